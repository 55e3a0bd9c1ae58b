// Per-row top-k select: T_t = Top-k(I_t) ("IndexCache: Accelerating Sparse
// Attention via Cross-Layer Index Reuse", notation of the method section;
// k = 2048 per §2.1).
//
// Output contract: the min(k, n) positions of the largest scores of a row,
// in ascending position order, ties going to the lower position, followed
// by -1 padding.  -0.0 and +0.0 compare equal.
//
// Algorithm (one 512-thread CTA per row), on order-preserving uint32 keys:
//  A. one pass: keys (staged in shared memory when the row fits) and a
//     2048-bin histogram of their top 11 bits;
//  B. the bin holding the k-th largest key is found by a block suffix scan;
//     the keys of that bin are compacted into a candidate list (usually a
//     small fraction of the row) and two more radix digits (11 + 10 bits)
//     are resolved on the candidates only.  If the bin is too large for
//     the list (massive ties), those digits are resolved on the full row.
//     Result: the threshold key T and krem, the number of keys equal to T
//     still to take;
//  C. each warp owns a contiguous segment of the row: it counts keys > T
//     and == T, one block scan turns the counts into output offsets, and a
//     second walk writes the selected positions in ascending order (a key
//     == T is selected while fewer than krem equal keys precede it).
// Rows that fit in shared memory are read from global memory once.
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSmemCap = 32768;  // scores per row staged in shared memory
constexpr int kCandCap = 4096;

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t b = __float_as_uint(x);
    if ((b & 0x7fffffffu) == 0) b = 0;  // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct TopkShared {
    uint32_t hist[2048];
    uint32_t cand[kCandCap];
    uint32_t wsum[kTopkWarps];
    uint32_t wcnt[2][kTopkWarps];
    uint32_t ncand;
    uint32_t bin;
    uint32_t above;
};

// Find the bin b (of nbins, 512 threads owning nbins/512 consecutive bins
// each) such that count(bins > b) < krem <= count(bins >= b).  Writes the
// bin and count(bins > b) to S.bin / S.above.  Must be called by all threads.
template <int NB>
__device__ __forceinline__ void find_bin(TopkShared& S, uint32_t krem) {
    constexpr int PER = NB / kTopkThreads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t c[PER], tot = 0;
#pragma unroll
    for (int b = 0; b < PER; ++b) {
        c[b] = S.hist[tid * PER + b];
        tot += c[b];
    }
    // inclusive suffix sum within the warp (higher lanes hold higher bins)
    uint32_t suf = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += v;
    }
    if (lane == 0) S.wsum[warp] = suf;  // the warp's total
    __syncthreads();
    uint32_t higher = 0;  // keys in the warps above this one
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w)
        if (w > warp) higher += S.wsum[w];
    const uint32_t incl = suf + higher;       // keys in bins >= my first bin
    const uint32_t above = incl - tot;        // keys in bins above mine
    if (above < krem && krem <= incl) {
        uint32_t acc = above;
#pragma unroll
        for (int b = PER - 1; b >= 0; --b) {
            if (acc + c[b] >= krem) {
                S.bin = tid * PER + b;
                S.above = acc;
                break;
            }
            acc += c[b];
        }
    }
    __syncthreads();
}

template <bool IN_SMEM>
__global__ void __launch_bounds__(kTopkThreads)
    k_topk(const float* __restrict__ scores, long long ld, int row0, int k, int causal_base,
           const int32_t* __restrict__ row_len, int32_t* __restrict__ out, long long ld_out) {
    extern __shared__ uint32_t srow[];
    __shared__ TopkShared S;

    const int r = row0 + blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = row_len ? row_len[r] : causal_base + r + 1;
    int32_t* o = out + static_cast<long long>(r) * ld_out;
    if (n <= k) {
        for (int i = tid; i < k; i += kTopkThreads) o[i] = i < n ? i : -1;
        return;
    }
    const float* row = scores + static_cast<long long>(r) * ld;
    auto key_at = [&](int i) -> uint32_t {
        return IN_SMEM ? srow[i] : order_key(__ldg(row + i));
    };

    // ---- A: keys + histogram of the top 11 bits
    for (int i = tid; i < 2048; i += kTopkThreads) S.hist[i] = 0;
    if (tid == 0) S.ncand = 0;
    __syncthreads();
    {
        const int n4 = n >> 2;
        const float4* row4 = reinterpret_cast<const float4*>(row);
        for (int i = tid; i < n4; i += kTopkThreads) {
            const float4 v = __ldg(row4 + i);
            const uint32_t u0 = order_key(v.x), u1 = order_key(v.y);
            const uint32_t u2 = order_key(v.z), u3 = order_key(v.w);
            if (IN_SMEM) *reinterpret_cast<uint4*>(srow + 4 * i) = make_uint4(u0, u1, u2, u3);
            atomicAdd(&S.hist[u0 >> 21], 1u);
            atomicAdd(&S.hist[u1 >> 21], 1u);
            atomicAdd(&S.hist[u2 >> 21], 1u);
            atomicAdd(&S.hist[u3 >> 21], 1u);
        }
        for (int i = 4 * n4 + tid; i < n; i += kTopkThreads) {
            const uint32_t u = order_key(__ldg(row + i));
            if (IN_SMEM) srow[i] = u;
            atomicAdd(&S.hist[u >> 21], 1u);
        }
    }
    __syncthreads();
    find_bin<2048>(S, static_cast<uint32_t>(k));
    const uint32_t b1 = S.bin;
    uint32_t krem = static_cast<uint32_t>(k) - S.above;
    const uint32_t in_bin = S.hist[b1];
    __syncthreads();  // everyone has read S.bin / S.above / S.hist[b1]

    // ---- B: resolve bits 20..10 and 9..0 within bin b1
    uint32_t prefix = b1 << 21, mask = 0xFFE00000u;
    const bool use_cand = in_bin <= static_cast<uint32_t>(kCandCap);
    if (use_cand) {
        for (int i = tid; i < n; i += kTopkThreads) {
            const uint32_t u = key_at(i);
            if ((u >> 21) == b1) S.cand[atomicAdd(&S.ncand, 1u)] = u;
        }
        __syncthreads();
    }
    const int ncand = use_cand ? static_cast<int>(S.ncand) : n;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        const uint32_t dmask = pass == 0 ? 0x7FFu : 0x3FFu;
        for (int i = tid; i < 2048; i += kTopkThreads) S.hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < ncand; i += kTopkThreads) {
            const uint32_t u = use_cand ? S.cand[i] : key_at(i);
            if ((u & mask) == prefix) atomicAdd(&S.hist[(u >> shift) & dmask], 1u);
        }
        __syncthreads();
        if (pass == 0)
            find_bin<2048>(S, krem);
        else
            find_bin<1024>(S, krem);
        prefix |= S.bin << shift;
        mask |= dmask << shift;
        krem -= S.above;
        __syncthreads();
    }
    const uint32_t T = prefix;

    // ---- C: per-warp segments, counts, offsets, ordered writes
    const int seg = ((n + kTopkWarps - 1) / kTopkWarps + 31) / 32 * 32;
    const int sb = warp * seg, se = min(n, sb + seg);
    uint32_t cg = 0, ce = 0;
    for (int base = sb; base < se; base += 32) {
        const int i = base + lane;
        uint32_t u = 0;
        if (i < se) u = key_at(i);
        const bool in = i < se;
        cg += __popc(__ballot_sync(0xffffffffu, in && u > T));
        ce += __popc(__ballot_sync(0xffffffffu, in && u == T));
    }
    if (lane == 0) {
        S.wcnt[0][warp] = cg;
        S.wcnt[1][warp] = ce;
    }
    __syncthreads();
    uint32_t G = 0, E = 0;
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w)
        if (w < warp) {
            G += S.wcnt[0][w];
            E += S.wcnt[1][w];
        }
    const unsigned lt = (1u << lane) - 1u;
    for (int base = sb; base < se; base += 32) {
        const int i = base + lane;
        uint32_t u = 0;
        if (i < se) u = key_at(i);
        const bool in = i < se;
        const bool gt = in && u > T, eq = in && u == T;
        const unsigned bg = __ballot_sync(0xffffffffu, gt);
        const unsigned be = __ballot_sync(0xffffffffu, eq);
        const uint32_t g_before = G + __popc(bg & lt);
        const uint32_t e_before = E + __popc(be & lt);
        if (gt)
            o[g_before + (e_before < krem ? e_before : krem)] = i;
        else if (eq && e_before < krem)
            o[g_before + e_before] = i;
        G += __popc(bg);
        E += __popc(be);
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
        const int smem = ((nmax < kTopkSmemCap ? nmax : kTopkSmemCap) + 3) / 4 * 16;
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
