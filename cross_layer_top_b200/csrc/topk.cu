// Per-row top-k select: T_t = Top-k(I_t) ("IndexCache: Accelerating Sparse
// Attention via Cross-Layer Index Reuse", notation of the method section;
// k = 2048 per §2.1).
//
// Output contract: the min(k, n) positions of the largest scores of a row,
// in ascending position order, ties going to the lower position, followed
// by -1 padding.  -0.0 and +0.0 compare equal.
//
// Algorithm (one 512-thread CTA per row):
//  1. Map each fp32 score to an order-preserving uint32 key.
//  2. Radix-select the k-th largest key with four 8-bit digit passes
//     (histograms in shared memory with warp-aggregated atomics; one warp
//     locates the digit whose bin crosses the remaining rank).  This yields
//     the threshold key T and `krem`, the number of keys equal to T that
//     are still to be taken.
//  3. One pass in position order: a key > T is selected; a key == T is
//     selected while fewer than krem equal keys precede it.  Ballots and a
//     block scan give each selected position its output slot, so the output
//     comes out ascending.
// Rows up to kSmemCap scores are staged in shared memory once (one global
// read); longer rows re-read global memory (L2) on every pass.
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSmemCap = 40960;  // scores per row kept in shared memory (160 KB)

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t b = __float_as_uint(x);
    if ((b & 0x7fffffffu) == 0) b = 0;  // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <bool IN_SMEM>
__global__ void __launch_bounds__(kTopkThreads)
    k_topk(const float* __restrict__ scores, long long ld, int row0, int k, int causal_base,
           const int32_t* __restrict__ row_len, int32_t* __restrict__ out, long long ld_out) {
    extern __shared__ uint32_t srow[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t wcnt[2][2][kTopkWarps];
    __shared__ uint32_t s_digit, s_above;

    const int r = row0 + blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = row_len ? row_len[r] : causal_base + r + 1;
    int32_t* o = out + static_cast<long long>(r) * ld_out;
    if (n <= k) {
        for (int i = tid; i < k; i += kTopkThreads) o[i] = i < n ? i : -1;
        return;
    }
    const float* row = scores + static_cast<long long>(r) * ld;
    if (IN_SMEM) {
        const int n4 = n >> 2;
        const float4* row4 = reinterpret_cast<const float4*>(row);
        for (int i = tid; i < n4; i += kTopkThreads) {
            const float4 v = __ldg(row4 + i);
            srow[4 * i + 0] = order_key(v.x);
            srow[4 * i + 1] = order_key(v.y);
            srow[4 * i + 2] = order_key(v.z);
            srow[4 * i + 3] = order_key(v.w);
        }
        for (int i = 4 * n4 + tid; i < n; i += kTopkThreads) srow[i] = order_key(__ldg(row + i));
        __syncthreads();
    }

    uint32_t prefix = 0, mask = 0;
    int krem = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += kTopkThreads) {
            const int i = base + tid;
            bool part = false;
            uint32_t digit = 0;
            if (i < n) {
                const uint32_t u = IN_SMEM ? srow[i] : order_key(__ldg(row + i));
                part = (u & mask) == prefix;
                digit = (u >> shift) & 255u;
            }
            const unsigned am = __ballot_sync(0xffffffffu, part);
            if (part) {
                const unsigned peers = __match_any_sync(am, digit);
                if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
            }
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns bins 8l .. 8l+7; find the bin where the count of
            // keys above crosses krem, scanning from the top bin down
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                c[b] = hist[8 * lane + b];
                tot += c[b];
            }
            // inclusive suffix sum over lanes (higher lanes hold higher bins)
            uint32_t suf = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t v = __shfl_down_sync(0xffffffffu, suf, off);
                if (lane + off < 32) suf += v;
            }
            const uint32_t above = suf - tot;  // keys in bins of higher lanes
            if (above < static_cast<uint32_t>(krem) && static_cast<uint32_t>(krem) <= suf) {
                uint32_t acc = above;
                for (int b = 7; b >= 0; --b) {
                    if (acc + c[b] >= static_cast<uint32_t>(krem)) {
                        s_digit = 8 * lane + b;
                        s_above = acc;
                        break;
                    }
                    acc += c[b];
                }
            }
        }
        __syncthreads();
        prefix |= s_digit << shift;
        mask |= 255u << shift;
        krem -= static_cast<int>(s_above);
    }
    const uint32_t T = prefix;

    // position-ordered compaction
    const unsigned lt = (1u << lane) - 1u;
    uint32_t G = 0, E = 0;  // selected-greater and equal counts before this tile
    int buf = 0;
    for (int base = 0; base < n; base += kTopkThreads) {
        const int i = base + tid;
        bool gt = false, eq = false;
        if (i < n) {
            const uint32_t u = IN_SMEM ? srow[i] : order_key(__ldg(row + i));
            gt = u > T;
            eq = u == T;
        }
        const unsigned bg = __ballot_sync(0xffffffffu, gt);
        const unsigned be = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) {
            wcnt[buf][0][warp] = __popc(bg);
            wcnt[buf][1][warp] = __popc(be);
        }
        __syncthreads();
        uint32_t wg = 0, we = 0, tg = 0, te = 0;
#pragma unroll
        for (int x = 0; x < kTopkWarps; ++x) {
            const uint32_t a = wcnt[buf][0][x], b = wcnt[buf][1][x];
            if (x < warp) {
                wg += a;
                we += b;
            }
            tg += a;
            te += b;
        }
        const uint32_t g_before = G + wg + __popc(bg & lt);
        const uint32_t e_before = E + we + __popc(be & lt);
        const uint32_t kr = static_cast<uint32_t>(krem);
        if (gt) {
            o[g_before + (e_before < kr ? e_before : kr)] = i;
        } else if (eq && e_before < kr) {
            o[g_before + e_before] = i;
        }
        G += tg;
        E += te;
        buf ^= 1;
    }
    // n > k here, so exactly k positions were written; nothing to pad.
}

int launch_topk(ic_ctx* ctx, const float* scores, int64_t ld, int rows, int k, int causal_base,
                const int32_t* row_len, int max_len, int32_t* idx_out, int64_t ld_out,
                cudaStream_t stream) {
    if (rows <= 0) return IC_OK;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_topk<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kTopkSmemCap * 4);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaFuncSetAttribute(topk)");
        attr_set = true;
    }
    // Causal rows r have n = causal_base + r + 1: rows whose n fits in shared
    // memory take the staged kernel, the rest the global-memory kernel.
    int split = rows;  // rows [0, split) staged, [split, rows) global
    if (row_len == nullptr) {
        const long long fit = static_cast<long long>(kTopkSmemCap) - causal_base;  // n <= cap
        split = fit < 0 ? 0 : (fit > rows ? rows : static_cast<int>(fit));
    } else if (max_len > kTopkSmemCap) {
        split = 0;
    }
    if (split > 0) {
        const int nmax = row_len ? max_len : causal_base + split;
        const int smem = (nmax < kTopkSmemCap ? nmax : kTopkSmemCap) * 4;
        LaunchScope ls(ctx, IC_K_TOPK, stream);
        k_topk<true><<<split, kTopkThreads, smem, stream>>>(scores, ld, 0, k, causal_base, row_len,
                                                             idx_out, ld_out);
        cudaError_t e = ls.done();
        if (e != cudaSuccess) return cuda_fail(ctx, e, "topk launch");
    }
    if (split < rows) {
        LaunchScope ls(ctx, IC_K_TOPK, stream);
        k_topk<false><<<rows - split, kTopkThreads, 0, stream>>>(scores, ld, split, k, causal_base,
                                                                 row_len, idx_out, ld_out);
        cudaError_t e = ls.done();
        if (e != cudaSuccess) return cuda_fail(ctx, e, "topk launch");
    }
    return IC_OK;
}

}  // namespace ic
