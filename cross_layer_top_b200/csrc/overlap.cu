// Cross-layer index overlap, the diagnostic behind index reuse: for two
// index tensors of the same query rows (the top-k sets T_a, T_b of two
// layers), hits[r] = |T_a[r] ∩ T_b[r]|, the overlap being hits / k ("IndexCache:
// Accelerating Sparse Attention via Cross-Layer Index Reuse", Appendix A;
// "IndexCache：跨层复用稀疏索引，以及它为什么能被训练", §3.2).
//
// One CTA per row.  Row r of b is marked in a shared-memory map over the key
// positions [0, n_keys) -- one byte per key when that fits (plain stores:
// every writer stores the same 1), else one bit (atomic OR); each valid entry
// of row r of a then tests its mark.  Entries -1 never count; an entry outside [-1, n_keys) is skipped and
// latched as a device error.  An entry of a counts once for each time it
// occurs in a, and an entry of b counts once however often it occurs, the
// same as a direct pairwise search.  The rows may be in any order.
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

constexpr int kOverlapThreads = 256;
constexpr int kOverlapMaxKeys = 32 * (200 * 1024 / 4);  // bitmap of at most 200 KB

constexpr int kOverlapByteMapKeys = 48 * 1024;

template <bool BYTES>
__global__ void __launch_bounds__(kOverlapThreads)
    k_index_overlap(const int32_t* __restrict__ a, const int32_t* __restrict__ b, int k, int n_keys,
                    int32_t* __restrict__ hits, int* __restrict__ err) {
    extern __shared__ uint32_t bits[];  // [ceil(n_keys / 32)] bits, or [ceil(n_keys / 4)] bytes
    __shared__ int warp_sum[kOverlapThreads / 32];
    uint8_t* bytes = reinterpret_cast<uint8_t*>(bits);
    const int r = blockIdx.x;
    const int nw = BYTES ? (n_keys + 3) >> 2 : (n_keys + 31) >> 5;
    for (int i = threadIdx.x; i < nw; i += kOverlapThreads) bits[i] = 0;
    __syncthreads();
    const int32_t* ar = a + static_cast<long long>(r) * k;
    const int32_t* br = b + static_cast<long long>(r) * k;
    // the first kPer entries of a and of b per thread are loaded at once, so a
    // row costs one memory round trip when k <= kPer * threads
    constexpr int kPer = 8;
    int av[kPer], bv[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kOverlapThreads;
        av[u] = i < k ? __ldg(ar + i) : -1;
        bv[u] = i < k ? __ldg(br + i) : -1;
    }
    bool bad = false;
    auto mark = [&](int v) {
        if (static_cast<unsigned>(v) < static_cast<unsigned>(n_keys)) {
            if (BYTES)
                bytes[v] = 1;
            else
                atomicOr(&bits[v >> 5], 1u << (v & 31));
        } else if (v != -1) {
            bad = true;
        }
    };
#pragma unroll
    for (int u = 0; u < kPer; ++u) mark(bv[u]);
    for (int i = threadIdx.x + kPer * kOverlapThreads; i < k; i += kOverlapThreads) mark(__ldg(br + i));
    __syncthreads();
    int cnt = 0;
    auto test = [&](int v) {
        if (static_cast<unsigned>(v) < static_cast<unsigned>(n_keys))
            cnt += BYTES ? bytes[v] : (bits[v >> 5] >> (v & 31)) & 1u;
        else if (v != -1)
            bad = true;
    };
#pragma unroll
    for (int u = 0; u < kPer; ++u) test(av[u]);
    for (int i = threadIdx.x + kPer * kOverlapThreads; i < k; i += kOverlapThreads) test(__ldg(ar + i));
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicCAS(err, 0, kDevBadIndex);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        int t = 0;
#pragma unroll
        for (int w = 0; w < kOverlapThreads / 32; ++w) t += warp_sum[w];
        hits[r] = t;
    }
}

int launch_index_overlap(ic_ctx* ctx, const int32_t* a, const int32_t* b, int rows, int k,
                         int n_keys, int32_t* hits, cudaStream_t stream) {
    if (n_keys > kOverlapMaxKeys)
        return fail(ctx, IC_ERR_UNSUPPORTED, "index_overlap: n_keys=%d (at most %d)", n_keys,
                    kOverlapMaxKeys);
    const bool byte_map = n_keys <= kOverlapByteMapKeys;
    const int smem = byte_map ? ((n_keys + 3) >> 2) * 4 : ((n_keys + 31) >> 5) * 4;
    // the bit-map form's shared memory grows with n_keys: its limit is raised
    // once per device to the largest map this kernel can need
    static PerDeviceOnce attr_once;
    if (!byte_map) {
        cudaError_t e = attr_once.run(ctx->device, [] {
            return cudaFuncSetAttribute(k_index_overlap<false>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        ((kOverlapMaxKeys + 31) >> 5) * 4);
        });
        if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaFuncSetAttribute(index_overlap)");
    }
    LaunchScope ls(ctx, IC_K_OVERLAP, stream);
    if (byte_map)
        k_index_overlap<true><<<rows, kOverlapThreads, smem, stream>>>(a, b, k, n_keys, hits,
                                                                      ctx->dev_err);
    else
        k_index_overlap<false><<<rows, kOverlapThreads, smem, stream>>>(a, b, k, n_keys, hits,
                                                                       ctx->dev_err);
    cudaError_t e = ls.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "index_overlap launch");
    return IC_OK;
}

}  // namespace ic
