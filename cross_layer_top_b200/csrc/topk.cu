// Per-row top-k select: T_t = Top-k(I_t) ("IndexCache: Accelerating Sparse
// Attention via Cross-Layer Index Reuse", notation of the method section;
// k = 2048 per §2.1).
//
// Output contract: the min(k, n) positions of the largest scores of a row,
// in ascending position order, ties going to the lower position, followed
// by -1 padding.  -0.0 and +0.0 compare equal.
//
// Algorithm (one CTA per row: 8 warps for rows up to 32768 keys, 16 warps
// beyond), on order-preserving uint32 keys:
//  A. one pass over the row: a 2048-bin histogram of the keys' top 11 bits;
//     the bin b1 holding the k-th largest key is found by a block suffix
//     scan;
//  B. a second pass, each warp over a contiguous segment: the ballot of
//     "bin above b1" is stored as a 32-bit word of a shared selection bitmap
//     (those keys are selected whatever the threshold), and the keys of bin
//     b1 go with their positions to the warp's own slice of a candidate
//     list.  Two more radix digits (11 + 10 bits) are resolved on the
//     candidates: the threshold key T and krem, the number of keys equal to
//     T still to take (the third digit is skipped when the second digit's
//     bin is taken whole: T is then that bin's smallest key);
//  C. when every key equal to T is taken (no tie split), the candidates
//     >= T are OR-ed into the bitmap and its set positions are gathered in
//     ascending order in shared memory (a block scan of the words'
//     popcounts gives each thread its offset), then written with coalesced
//     stores.  Otherwise (a tie split, a candidate bin too large
//     for the list, or a row longer than the bitmap) the general path:
//     digits resolved on the full row, then per-warp counts of keys > T and
//     == T, a block scan, and an ordered walk that takes a key == T while
//     fewer than krem equal keys precede it.
// The row is read from global memory twice (L2 holds it between the passes).
#include <cstddef>

#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

// cluster variant: 16 warps per CTA, 4096 candidate slots
constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kCandCap = 4096;
// single-CTA row kernel, two shapes:
//  - rows up to kShortRow keys: 8 warps per CTA and 2048 candidate slots, so
//    eight CTAs share an SM at 16K keys (measured on one prefill F layer's
//    14336 rows: 0.379 ms against 0.411 ms with the long-row shape; 8 warps
//    with 4096 slots and four CTAs per SM gained nothing);
//  - longer rows: 16 warps and 4096 slots.  On Gaussian scores the bin of
//    the k-th largest key holds about 2170 keys at 131072 keys, which the
//    short-row list would send to the general path.
constexpr int kShortRow = 32768;
constexpr int kBitmapCap = 131072;  // longest row (keys) with a shared selection bitmap

// inverse of order_key (up to the sign of zero)
__device__ __forceinline__ float key_float(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// hist and cand are read with 16-byte (remote) loads in the cluster variant
template <int WARPS, int CAND>
struct alignas(16) TopkSharedT {
    static constexpr int kWarps = WARPS;
    alignas(16) uint32_t hist[2048];
    alignas(16) uint32_t cand[CAND];
    uint32_t wsum[WARPS];
    uint32_t wcnt[2][WARPS];
    uint32_t ncand;
    uint32_t wcand[WARPS];  // bitmap path: candidates in each warp's slice
    uint32_t bin;
    uint32_t above;
    uint32_t bin_count;  // keys in `bin`
};
using TopkShared = TopkSharedT<kTopkWarps, kCandCap>;

// Find the bin b (of NB, the CTA's threads owning NB / threads consecutive
// bins each) such that count(bins > b) < krem <= count(bins >= b).  Writes
// the bin and count(bins > b) to S.bin / S.above.  Must be called by all
// threads.  This form takes the thread's counts of bins tid*PER ..
// tid*PER+PER-1 in registers and also writes the found bin's count to
// S.bin_count.
template <int NB, class SH>
__device__ __forceinline__ void find_bin_counts(SH& S, uint32_t krem,
                                                const uint32_t (&c)[NB / (SH::kWarps * 32)]) {
    constexpr int WARPS = SH::kWarps;
    constexpr int PER = NB / (WARPS * 32);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t tot = 0;
#pragma unroll
    for (int b = 0; b < PER; ++b) tot += c[b];
    // inclusive suffix sum within the warp (higher lanes hold higher bins)
    uint32_t suf = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += v;
    }
    if (lane == 0) S.wsum[warp] = suf;  // the warp's total
    __syncthreads();
    // keys in the warps above this one: a suffix scan of the warp totals
    // across lanes (lane w ends with the keys in warps >= w; lanes past the
    // last warp hold 0)
    uint32_t ws = lane < WARPS ? S.wsum[lane] : 0u;
#pragma unroll
    for (int off = 1; off < WARPS; off <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, ws, off);
        if (lane + off < WARPS) ws += v;
    }
    const uint32_t higher = __shfl_sync(0xffffffffu, ws, warp + 1);
    const uint32_t incl = suf + higher;       // keys in bins >= my first bin
    const uint32_t above = incl - tot;        // keys in bins above mine
    if (above < krem && krem <= incl) {
        uint32_t acc = above;
#pragma unroll
        for (int b = PER - 1; b >= 0; --b) {
            if (acc + c[b] >= krem) {
                S.bin = tid * PER + b;
                S.above = acc;
                S.bin_count = c[b];
                break;
            }
            acc += c[b];
        }
    }
    __syncthreads();
}
template <int NB, class SH>
__device__ __forceinline__ void find_bin(SH& S, uint32_t krem, const uint32_t* hist) {
    constexpr int PER = NB / (SH::kWarps * 32);
    uint32_t c[PER];
#pragma unroll
    for (int b = 0; b < PER; ++b) c[b] = hist[threadIdx.x * PER + b];
    find_bin_counts<NB>(S, krem, c);
}
template <int NB, class SH>
__device__ __forceinline__ void find_bin(SH& S, uint32_t krem) {
    find_bin<NB>(S, krem, S.hist);
}

template <int kRowThreads, int kRowCandCap, int kRowMinCtas>
__global__ void __launch_bounds__(kRowThreads, kRowMinCtas)
    k_topk(const float* __restrict__ scores, long long ld, int k, int causal_base,
           const int32_t* __restrict__ row_len, int max_len, int32_t* __restrict__ out,
           long long ld_out, int bcap) {
    // dynamic shared memory: the candidates' positions [kRowCandCap], then the
    // selection bitmap of rows up to bcap keys [bcap / 32]
    extern __shared__ uint32_t dsm[];
    constexpr int kRowWarps = kRowThreads / 32;
    __shared__ TopkSharedT<kRowWarps, kRowCandCap> S;

    const int r = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // as a programmatic dependent: nothing is read before the previous kernel completes
    griddep_wait();
    griddep_launch_dependents();
    // a given length above max_len (the row stride) counts as max_len
    const int n = row_len ? min(row_len[r], max_len) : causal_base + r + 1;
    int32_t* o = out + static_cast<long long>(r) * ld_out;
    if (n <= k) {
        for (int i = tid; i < k; i += kRowThreads) o[i] = i < n ? i : -1;
        return;
    }
    const float* row = scores + static_cast<long long>(r) * ld;
    auto key_at = [&](int i) -> uint32_t { return order_key(__ldg(row + i)); };
    // ---- A: histogram of the keys' top 11 bits.  It is counted on the raw
    // float bits: raw top bits r lie in key bin r + 1024 (r < 1024) or
    // 2047 - r, for every score but -0.0, whose raw bits fall in bin 1023
    // while its key (that of +0.0) is in bin 1024.  Only a threshold in bin
    // 1023 or 1024 depends on that: such a row is counted again on keys.
    auto count_keys = [&](bool raw) {
        for (int i = tid; i < 2048; i += kRowThreads) S.hist[i] = 0;
        __syncthreads();
        const int n4 = n >> 2;
        const float4* row4 = reinterpret_cast<const float4*>(row);
        auto bin = [&](float x) { return (raw ? __float_as_uint(x) : order_key(x)) >> 21; };
        for (int i = tid; i < n4; i += kRowThreads) {
            const float4 v = __ldg(row4 + i);
            atomicAdd(&S.hist[bin(v.x)], 1u);
            atomicAdd(&S.hist[bin(v.y)], 1u);
            atomicAdd(&S.hist[bin(v.z)], 1u);
            atomicAdd(&S.hist[bin(v.w)], 1u);
        }
        for (int i = 4 * n4 + tid; i < n; i += kRowThreads) atomicAdd(&S.hist[bin(__ldg(row + i))], 1u);
        __syncthreads();
        constexpr int PER = 2048 / kRowThreads;
        uint32_t c[PER];
#pragma unroll
        for (int b = 0; b < PER; ++b) {
            const int key_bin = tid * PER + b;
            c[b] = S.hist[!raw ? key_bin : (key_bin >= 1024 ? key_bin - 1024 : 2047 - key_bin)];
        }
        find_bin_counts<2048>(S, static_cast<uint32_t>(k), c);
    };
    if (tid == 0) S.ncand = 0;
    count_keys(true);
    if (S.bin == 1023u || S.bin == 1024u) {  // the same in every thread
        __syncthreads();  // everyone has read S.bin
        count_keys(false);
    }
    const uint32_t b1 = S.bin;
    uint32_t krem = static_cast<uint32_t>(k) - S.above;
    const uint32_t in_bin = S.bin_count;
    __syncthreads();  // everyone has read S.bin / S.above / S.bin_count

    // ---- B: resolve bits 20..10 and 9..0 within bin b1
    uint32_t prefix = b1 << 21, mask = 0xFFE00000u;
    const bool use_cand = in_bin <= static_cast<uint32_t>(kRowCandCap);
    // warp segments, whole 128-key blocks (a warp's float4 load of 4 keys per lane)
    const int seg = ((n + kRowWarps - 1) / kRowWarps + 127) / 128 * 128;
    const int sb = warp * seg, se = min(n, sb + seg);
    const unsigned lt = (1u << lane) - 1u;
    uint32_t* cpos = dsm;
    uint32_t* bits = cpos + kRowCandCap;
    constexpr int kSlice = kRowCandCap / kRowWarps;  // candidate slots per warp
    bool sliced = false;  // candidates in per-warp slices of the list, bitmap path
    if (use_cand && n <= bcap) {
        // one pass over the warp's segment: the keys above bin b1 (selected
        // whatever T is) become bitmap words straight from the ballot; the
        // keys of bin b1 go to the warp's own slice of the candidate list
        // with their positions (a count in registers: no shared atomics)
        // Lane l takes keys base + 4l .. base + 4l + 3 (one float4; the row
        // start is 16-byte aligned and its stride a multiple of 4 floats, so
        // a load that starts before n stays inside the row's storage).
        uint32_t wc = 0;
        for (int base = sb; base < se; base += 128) {
            const int i0 = base + 4 * lane;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i0 < se) v = __ldg(reinterpret_cast<const float4*>(row + i0));
            const float x[4] = {v.x, v.y, v.z, v.w};
            uint32_t u[4], nib = 0;
            bool c[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool in = i0 + j < se;
                u[j] = order_key(x[j]);
                const uint32_t bin = u[j] >> 21;
                nib |= static_cast<uint32_t>(in && bin > b1) << j;
                c[j] = in && bin == b1;
            }
            // bitmap word m of the block holds lanes 8m .. 8m+7's nibbles
            uint32_t word = nib << (4 * (lane & 7));
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            word |= __shfl_xor_sync(0xffffffffu, word, 2);
            word |= __shfl_xor_sync(0xffffffffu, word, 4);
            if ((lane & 7) == 0 && base + 4 * lane < se) bits[(base >> 5) + (lane >> 3)] = word;
            // keys of bin b1: this lane's slots follow the lower lanes' (all j)
            unsigned bc[4];
            uint32_t j0 = wc;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bc[j] = __ballot_sync(0xffffffffu, c[j]);
                j0 += __popc(bc[j] & lt);
                wc += __popc(bc[j]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (c[j]) {
                    if (j0 < static_cast<uint32_t>(kSlice)) {
                        S.cand[warp * kSlice + j0] = u[j];
                        cpos[warp * kSlice + j0] = static_cast<uint32_t>(i0 + j);
                    }
                    ++j0;
                }
            }
        }
        if (lane == 0) S.wcand[warp] = wc;
        __syncthreads();
        bool over = false;  // a slice overflowed: take the general path
#pragma unroll
        for (int w = 0; w < kRowWarps; ++w) over |= S.wcand[w] > static_cast<uint32_t>(kSlice);
        sliced = !over;
    }
    if (use_cand && !sliced) {
        for (int i = tid; i < n; i += kRowThreads) {
            const uint32_t u = key_at(i);
            if ((u >> 21) == b1) S.cand[atomicAdd(&S.ncand, 1u)] = u;
        }
        __syncthreads();
    }
    const int ncand = use_cand ? static_cast<int>(S.ncand) : n;
    // sliced: each warp walks its own slice; otherwise the threads stride the list (or row)
    const int c0 = sliced ? warp * kSlice + lane : tid;
    const int c1 = sliced ? warp * kSlice + static_cast<int>(S.wcand[warp]) : ncand;
    const int cstep = sliced ? 32 : kRowThreads;
    // On the bitmap path the third digit is skipped when the second
    // digit's bin is taken whole (the usual case for real-valued scores):
    // T is then that bin's smallest key, and the keys >= T are exactly the
    // selection.
    bool whole = false;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        const uint32_t dmask = pass == 0 ? 0x7FFu : 0x3FFu;
        for (int i = tid; i < 2048; i += kRowThreads) S.hist[i] = 0;
        __syncthreads();
        for (int i = c0; i < c1; i += cstep) {
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
        const bool taken_whole = pass == 0 && sliced && krem == S.bin_count;  // the same in every thread
        __syncthreads();
        if (taken_whole) {
            whole = true;
            break;
        }
    }
    const uint32_t T = prefix;

    // ---- C (bitmap): when every key equal to T is taken, mark the
    // candidates >= T in the bitmap, gather its set positions in order in
    // shared memory (over the candidates' positions, no longer needed),
    // then write the row's k positions with coalesced stores
    if (sliced && (whole || krem == S.hist[T & 0x3FFu])) {
        for (int j = c0; j < c1; j += 32)
            if (S.cand[j] >= T) {
                const int pos = cpos[j];
                atomicOr(&bits[pos >> 5], 1u << (pos & 31));
            }
        __syncthreads();
        const int nw = (n + 31) >> 5;
        const int wpt = (nw + kRowThreads - 1) / kRowThreads;  // words per thread
        const int w0 = min(nw, tid * wpt), w1 = min(nw, w0 + wpt);
        uint32_t cnt = 0;
        for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
        uint32_t incl = cnt;  // inclusive scan of the counts in thread order
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) S.wsum[warp] = incl;
        __syncthreads();
        // positions in the warps before this one: a prefix scan of the warp
        // totals across lanes (lane w ends with the positions in warps <= w)
        uint32_t ws = lane < kRowWarps ? S.wsum[lane] : 0u;
#pragma unroll
        for (int off = 1; off < kRowWarps; off <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, ws, off);
            if (lane >= off) ws += v;
        }
        const uint32_t before = __shfl_sync(0xffffffffu, ws, warp > 0 ? warp - 1 : 0);
        uint32_t at = incl - cnt + (warp > 0 ? before : 0u);
        uint32_t* opos = cpos;  // k <= kRowCandCap slots
        for (int w = w0; w < w1; ++w)
            for (uint32_t x = bits[w]; x; x &= x - 1u) {
                // exactly k bits are set; the bound only guards the buffer
                if (at < static_cast<uint32_t>(k)) opos[at] = (w << 5) + (__ffs(x) - 1);
                ++at;
            }
        __syncthreads();
        for (int i = tid; i < k; i += kRowThreads) o[i] = static_cast<int32_t>(opos[i]);
        return;
    }

    // ---- C (ordered passes): per-warp segments, counts, offsets, writes
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
    for (int w = 0; w < kRowWarps; ++w)
        if (w < warp) {
            G += S.wcnt[0][w];
            E += S.wcnt[1][w];
        }
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

// ------------------------------------------------------------------------
// Cluster variant for few long rows (the decode step: B rows of up to
// ~200K candidates).  One thread-block cluster of kClusterCtas CTAs per row;
// CTA `rank` stages the row segment [rank*seg, (rank+1)*seg) in its shared
// memory (one bulk copy).  With the scan's first-digit histogram of the row
// the bin b1 of the k-th largest key is known before the row is read, and
// its keys form a short candidate list; without it, a first-level
// histogram of 2048 bins uniform in VALUE between the row's min and max (a
// monotone function of the score, so every key in a higher bin is larger)
// narrows bin b1.  The row-wide quantities (min/max, histograms, candidate
// lists, per-segment counts) are exchanged through distributed shared
// memory (mapa + ld.shared::cluster) between cluster barriers; every CTA
// then takes the same decisions, and each writes the selected positions of
// its own segment (through a selection bitmap when every key equal to the
// threshold is taken) at the offsets of the segments before it.  Same
// output contract as k_topk.
constexpr int kClusterCtas = 8;

struct alignas(16) TopkClusterShared {
    TopkShared S;
    alignas(16) uint32_t hist_all[2048];
    // pushed by each CTA q into the others' copies (slot q): its segment's
    // key range, and (for the later segments) its counts of keys > T and == T
    uint32_t rng_min[kClusterCtas], rng_max[kClusterCtas];
    uint32_t cnt_g[kClusterCtas], cnt_e[kClusterCtas];
    alignas(8) uint64_t stage_bar;  // completion of the segment's bulk copy
};
static_assert(offsetof(TopkShared, hist) % 16 == 0 && offsetof(TopkShared, cand) % 16 == 0,
              "16-byte loads of the histogram and candidates");
static_assert(offsetof(TopkClusterShared, hist_all) % 16 == 0, "16-byte stores of hist_all");

__global__ void __launch_bounds__(kTopkThreads)
    k_topk_cluster(const float* __restrict__ scores, long long ld, int k,
                   const int32_t* __restrict__ row_len, int max_len, int causal_base,
                   int32_t* __restrict__ out, long long ld_out, int seg_cap,
                   uint32_t* __restrict__ ghist, int* __restrict__ err) {
    // dynamic shared memory: the staged segment, then the merged candidates
    extern __shared__ uint32_t srow[];
    uint32_t* cand_all = srow + seg_cap;
    __shared__ TopkClusterShared CS;
    TopkShared& S = CS.S;
    const int r = blockIdx.y;
    const uint32_t rank = cluster_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // as a programmatic dependent: nothing is read before the previous kernel completes
    griddep_wait();
    griddep_launch_dependents();
    const int n = row_len ? min(row_len[r], max_len) : causal_base + r + 1;
    int32_t* o = out + static_cast<long long>(r) * ld_out;
    // the row's first-digit histogram from the scan, if given; CTA 0 clears
    // it once every CTA of the cluster is past reading it
    uint32_t* gh = ghist ? ghist + static_cast<long long>(r) * kKeyBins : nullptr;
    auto clear_hist = [&]() {
        if (gh != nullptr && rank == 0)
            for (int i = tid; i < kKeyBins; i += kTopkThreads) gh[i] = 0u;
    };
    if (n <= k) {  // the same for every CTA of the cluster: no cluster barrier is reached
        if (rank == 0)
            for (int i = tid; i < k; i += kTopkThreads) o[i] = i < n ? i : -1;
        clear_hist();
        return;
    }
    // With the histogram: the bin b1 of the k-th largest key and how many
    // keys it holds are known before the row is read.  If they fit the
    // candidate list (the same answer in every CTA), each CTA stages its
    // segment and collects the keys of bin b1 in one pass, and the radix
    // passes start at the second digit; otherwise the path below.
    const int seg = ((n + kClusterCtas - 1) / kClusterCtas + 3) / 4 * 4;
    const int s0 = min(n, static_cast<int>(rank) * seg), s1 = min(n, s0 + seg);
    const int m = s1 - s0;  // this CTA's segment length
    const float* row = scores + static_cast<long long>(r) * ld + s0;
    // this segment as order keys in shared memory; returns the segment's
    // key range (the path without a histogram needs it)
    auto stage = [&](uint32_t& kmin, uint32_t& kmax) {
        kmin = 0xFFFFFFFFu;
        kmax = 0u;
        // The segment's whole float4s arrive by one bulk copy that completes
        // on an mbarrier (the row start and the segment start are 16-byte
        // aligned; at most 45000 keys, within the transaction count), the
        // last m mod 4 scores by plain loads; then every float becomes its
        // order key in place.
        const int m4 = m >> 2;
        const uint32_t bytes = static_cast<uint32_t>(m4) * 16u;
        if (tid == 0) {
            mbar_init(&CS.stage_bar, 1);
            fence_mbar_init();
        }
        __syncthreads();
        if (tid == 0 && bytes > 0) {
            mbar_arrive_expect_tx(&CS.stage_bar, bytes);
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                ::"r"(smem_u32(srow)), "l"(row), "r"(bytes), "r"(smem_u32(&CS.stage_bar))
                : "memory");
        }
        for (int i = 4 * m4 + tid; i < m; i += kTopkThreads) {
            const uint32_t u = order_key(__ldg(row + i));
            srow[i] = u;
            kmin = min(kmin, u);
            kmax = max(kmax, u);
        }
        if (bytes > 0 && !mbar_wait_drain(&CS.stage_bar, 0)) {
            // bounded: the keys are then not the row's; the error is latched
            if (tid == 0 && err != nullptr) atomicCAS(err, 0, kDevTimeoutProducer);
        }
        uint4* srow4 = reinterpret_cast<uint4*>(srow);
        for (int i = tid; i < m4; i += kTopkThreads) {
            const uint4 v = srow4[i];
            const uint32_t u0 = order_key(__uint_as_float(v.x)), u1 = order_key(__uint_as_float(v.y));
            const uint32_t u2 = order_key(__uint_as_float(v.z)), u3 = order_key(__uint_as_float(v.w));
            srow4[i] = make_uint4(u0, u1, u2, u3);
            kmin = min(kmin, min(min(u0, u1), min(u2, u3)));
            kmax = max(kmax, max(max(u0, u1), max(u2, u3)));
        }
    };
    // The histogram's counts are loaded before the segment, so that their
    // round trip overlaps the staging reads.
    bool fast = false;
    uint32_t fb1 = 0, fkrem = 0;
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    if (gh != nullptr) {
        uint32_t c[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) c[b] = gh[tid * 4 + b];
        stage(kmin, kmax);
        if (tid == 0) {  // defined even if the counts were not the row's (find_bin orders this)
            S.bin = 0;
            S.above = 0;
            S.bin_count = 0xFFFFFFFFu;
        }
        find_bin_counts<2048>(S, static_cast<uint32_t>(k), c);
        fb1 = S.bin;
        fkrem = static_cast<uint32_t>(k) - S.above;
        fast = S.bin_count <= static_cast<uint32_t>(kCandCap);  // the same in every CTA
        __syncthreads();  // S.bin / S.above are rewritten below
    }
    // every CTA's candidate count, then its candidates at the running offset:
    // 4 per 16-byte remote load, each round's loads (one per CTA) issued
    // before any is stored; returns the merged count
    auto merge_candidates = [&]() {
        int nq[kClusterCtas], off[kClusterCtas], total = 0;
#pragma unroll
        for (uint32_t q = 0; q < kClusterCtas; ++q) nq[q] = static_cast<int>(dsmem_ld(dsmem_addr(&S.ncand, q)));
#pragma unroll
        for (uint32_t q = 0; q < kClusterCtas; ++q) {
            nq[q] = min(nq[q], kCandCap - total);  // never past the merged list
            off[q] = total;
            total += nq[q];
        }
        for (int i4 = 4 * tid; i4 < kCandCap; i4 += 4 * kTopkThreads) {
            // two rounds of loads from half the CTAs each
#pragma unroll
            for (uint32_t h = 0; h < kClusterCtas; h += kClusterCtas / 2) {
                uint4 cv[kClusterCtas / 2];
#pragma unroll
                for (uint32_t q = 0; q < kClusterCtas / 2; ++q)
                    if (i4 < nq[h + q]) cv[q] = dsmem_ld_u4(dsmem_addr(&S.cand[i4], h + q));
#pragma unroll
                for (uint32_t q = 0; q < kClusterCtas / 2; ++q) {
                    const uint32_t c4[4] = {cv[q].x, cv[q].y, cv[q].z, cv[q].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (i4 + e < nq[h + q]) cand_all[off[h + q] + i4 + e] = c4[e];
                }
            }
        }
        // No CTA rewrites its S.ncand or S.cand after this, so other CTAs may
        // still be reading them: only this CTA's merged list must be complete.
        __syncthreads();
        return total;
    };
    uint32_t prefix = 0, mask = 0, krem = 0;
    bool use_cand = true;
    int ncand = 0, first_pass = 0;
    // The path without a histogram bins keys uniformly in value between the
    // row's minimum and maximum (monotone in the key, so exact), or by their
    // top 11 bits when that range is degenerate.
    float xmin = 0.f, inv = 0.f;
    bool by_value = false;
    uint32_t b1 = 0;
    auto bin_of = [&](uint32_t u) -> uint32_t {
        if (!by_value) return u >> 21;
        return static_cast<uint32_t>(fminf((key_float(u) - xmin) * inv, 2047.0f));
    };
    // cluster-wide histogram: local counts, then every CTA sums all of them
    // each thread sums 4 consecutive bins (2048 = 4 x 512) over the cluster's
    // CTAs with one 16-byte remote load per CTA, all issued before any is used
    static_assert(2048 == 4 * kTopkThreads, "four bins per thread");
    // rewrite_next: the caller rewrites its histogram right after (another
    // radix pass over the row), so a second barrier keeps every CTA's reads
    // of it ahead of that; otherwise a later cluster barrier does
    auto cluster_hist = [&](bool rewrite_next) {
        cluster_sync_all();  // every segment histogram is complete
        uint4 hv[kClusterCtas];
#pragma unroll
        for (uint32_t q = 0; q < kClusterCtas; ++q) hv[q] = dsmem_ld_u4(dsmem_addr(&S.hist[4 * tid], q));
        uint4 t = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (uint32_t q = 0; q < kClusterCtas; ++q) {
            t.x += hv[q].x;
            t.y += hv[q].y;
            t.z += hv[q].z;
            t.w += hv[q].w;
        }
        *reinterpret_cast<uint4*>(&CS.hist_all[4 * tid]) = t;
        if (rewrite_next) cluster_sync_all();  // nobody rewrites a histogram another CTA still reads
    };
    if (fast) {
        if (tid == 0) S.ncand = 0;
        __syncthreads();
        // four staged keys per 16-byte load (the staged segment's storage is
        // a multiple of 4 keys; keys past m are not the row's)
        for (int i4 = tid; 4 * i4 < m; i4 += kTopkThreads) {
            const uint4 v = *reinterpret_cast<const uint4*>(srow + 4 * i4);
            const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (4 * i4 + j < m && (u4[j] >> kKeyBinShift) == fb1) {
                    // the counts bound the list; the check only keeps counts
                    // that do not belong to these scores from writing past it
                    const uint32_t slot = atomicAdd(&S.ncand, 1u);
                    if (slot < static_cast<uint32_t>(kCandCap)) S.cand[slot] = u4[j];
                }
            }
        }
        // every CTA of the cluster is running and has its candidates, and
        // has read the histogram
        cluster_sync_all();
        clear_hist();
        ncand = merge_candidates();
        prefix = fb1 << kKeyBinShift;
        mask = 0x7FFu << kKeyBinShift;
        krem = fkrem;
        first_pass = 1;
    } else {
        // every CTA arrives on the cluster barrier now and waits on it before its
        // first remote store, by when the whole cluster is known to be running
        cluster_arrive_relaxed();

        // ---- A: stage the segment (unless done above), cluster-wide key range
        if (gh == nullptr) stage(kmin, kmax);
        kmin = __reduce_min_sync(0xffffffffu, kmin);
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0) {
            S.wcnt[0][warp] = kmin;
            S.wcnt[1][warp] = kmax;
        }
        for (int i = tid; i < 2048; i += kTopkThreads) S.hist[i] = 0;
        if (tid == 0) S.ncand = 0;
        __syncthreads();
        cluster_wait_acquire();  // every CTA of the cluster is running
        clear_hist();            // ... and past reading the histogram
        // thread q stores this segment's range into CTA q's slot `rank`
        if (tid < kClusterCtas) {
            uint32_t a = 0xFFFFFFFFu, b = 0u;
            for (int w = 0; w < kTopkWarps; ++w) {
                a = min(a, S.wcnt[0][w]);
                b = max(b, S.wcnt[1][w]);
            }
            dsmem_st_u32(dsmem_addr(&CS.rng_min[rank], tid), a);
            dsmem_st_u32(dsmem_addr(&CS.rng_max[rank], tid), b);
        }
        cluster_sync_all();  // every segment's range is in every CTA
        kmin = 0xFFFFFFFFu;
        kmax = 0u;
#pragma unroll
        for (int q = 0; q < kClusterCtas; ++q) {
            kmin = min(kmin, CS.rng_min[q]);
            kmax = max(kmax, CS.rng_max[q]);
        }
        xmin = key_float(kmin);
        const float span = key_float(kmax) - xmin;
        inv = 2047.0f / span;
        by_value = span > 0.f && isfinite(span) && isfinite(inv) && inv > 0.f;
        for (int i = tid; i < m; i += kTopkThreads) atomicAdd(&S.hist[bin_of(srow[i])], 1u);
        cluster_hist(false);
        find_bin<2048>(S, static_cast<uint32_t>(k), CS.hist_all);
        b1 = S.bin;
        krem = static_cast<uint32_t>(k) - S.above;
        const uint32_t in_bin = CS.hist_all[b1];
        __syncthreads();

        // ---- B: candidates of bin b1 from every segment, or (massive ties)
        // cluster-wide radix passes over the bin's keys
        use_cand = in_bin <= static_cast<uint32_t>(kCandCap);  // the same in every CTA
        // The radix passes rewrite S.hist.  With candidates, the barrier after
        // they are collected keeps every CTA's reads of the histograms above
        // ahead of that; without, this one does.
        if (!use_cand) cluster_sync_all();
        if (use_cand) {
            for (int i = tid; i < m; i += kTopkThreads) {
                const uint32_t u = srow[i];
                if (bin_of(u) == b1) S.cand[atomicAdd(&S.ncand, 1u)] = u;
            }
            cluster_sync_all();
            ncand = merge_candidates();
        }
    }  // the path without a histogram (or with too many keys in its bin)
    bool whole = false;  // the second digit's bin taken whole (below)
#pragma unroll 1
    for (int pass = first_pass; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
        for (int i = tid; i < 2048; i += kTopkThreads) S.hist[i] = 0;
        __syncthreads();
        if (use_cand) {
            for (int i = tid; i < ncand; i += kTopkThreads) {
                const uint32_t u = cand_all[i];
                if ((u & mask) == prefix) atomicAdd(&S.hist[(u >> shift) & dmask], 1u);
            }
            __syncthreads();
        } else {
            for (int i = tid; i < m; i += kTopkThreads) {
                const uint32_t u = srow[i];
                if ((u & mask) == prefix && bin_of(u) == b1)
                    atomicAdd(&S.hist[(u >> shift) & dmask], 1u);
            }
            cluster_hist(true);
        }
        const uint32_t* h = use_cand ? S.hist : CS.hist_all;
        if (pass < 2)
            find_bin<2048>(S, krem, h);
        else
            find_bin<1024>(S, krem, h);
        prefix |= S.bin << shift;
        mask |= dmask << shift;
        krem -= S.above;
        // the second digit's bin taken whole (the usual case): T = its
        // smallest key, every key >= T is selected and the third digit is
        // not needed (the same answer in every thread and CTA)
        const bool taken_whole = pass == 1 && use_cand && krem == S.bin_count;
        __syncthreads();
        if (taken_whole) {
            whole = true;
            break;
        }
    }
    const uint32_t T = prefix;

    // ---- C (bitmap): when every key equal to T is taken (the same answer in
    // every CTA: it follows from the merged candidates), the selection is
    // the keys >= T.  One pass marks this segment's keys >= T in a bitmap
    // (over the merged candidates, no longer needed), a block scan of the
    // words' popcounts gives each thread its offset, the segment's total goes
    // to the later CTAs, and the positions are gathered in order in shared
    // memory (over this CTA's candidate list, which no CTA reads after the
    // barrier) and written with coalesced stores.
    if (use_cand && (whole || krem == S.hist[T & 0x3FFu])) {
        uint32_t* bits = cand_all;  // ceil(m / 32) <= kCandCap words
        for (int base = 128 * warp; base < m; base += 128 * kTopkWarps) {
            const int i0 = base + 4 * lane;
            uint32_t nib = 0;
            if (i0 + 3 < m) {
                const uint4 v = *reinterpret_cast<const uint4*>(srow + i0);
                nib = static_cast<uint32_t>(v.x >= T) | static_cast<uint32_t>(v.y >= T) << 1 |
                      static_cast<uint32_t>(v.z >= T) << 2 | static_cast<uint32_t>(v.w >= T) << 3;
            } else {
                for (int j = 0; j < 4 && i0 + j < m; ++j)
                    nib |= static_cast<uint32_t>(srow[i0 + j] >= T) << j;
            }
            // word w of the block holds lanes 8w .. 8w+7's nibbles
            uint32_t word = nib << (4 * (lane & 7));
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            word |= __shfl_xor_sync(0xffffffffu, word, 2);
            word |= __shfl_xor_sync(0xffffffffu, word, 4);
            if ((lane & 7) == 0 && i0 < m) bits[(base >> 5) + (lane >> 3)] = word;
        }
        __syncthreads();
        const int nw = (m + 31) >> 5;
        const int wpt = (nw + kTopkThreads - 1) / kTopkThreads;  // words per thread
        const int w0 = min(nw, tid * wpt), w1 = min(nw, w0 + wpt);
        uint32_t cnt = 0;
        for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
        uint32_t incl = cnt;  // inclusive scan of the counts in thread order
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += x;
        }
        if (lane == 31) S.wsum[warp] = incl;
        __syncthreads();
        // positions in the warps before this one, and the segment's total
        uint32_t ws = lane < kTopkWarps ? S.wsum[lane] : 0u;
#pragma unroll
        for (int off = 1; off < kTopkWarps; off <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, ws, off);
            if (lane >= off) ws += x;
        }
        const uint32_t before = __shfl_sync(0xffffffffu, ws, warp > 0 ? warp - 1 : 0);
        const uint32_t total = __shfl_sync(0xffffffffu, ws, kTopkWarps - 1);
        // thread q > rank stores this segment's total into CTA q's slot `rank`
        if (tid < kClusterCtas && tid > static_cast<int>(rank))
            dsmem_st_u32(dsmem_addr(&CS.cnt_g[rank], tid), total);
        // The last cluster barrier, as on the path below.
        cluster_sync_all();
        uint32_t G = 0;  // selected positions in the segments before this one
        for (uint32_t q = 0; q < rank; ++q) G += CS.cnt_g[q];
        uint32_t at = incl - cnt + (warp > 0 ? before : 0u);
        uint32_t* opos = S.cand;
        for (int w = w0; w < w1; ++w)
            for (uint32_t x = bits[w]; x; x &= x - 1u) {
                // the segment holds at most k selected keys; the bound only
                // guards the buffer against counts that were not the row's
                if (at < static_cast<uint32_t>(kCandCap))
                    opos[at] = static_cast<uint32_t>(s0 + (w << 5) + (__ffs(x) - 1));
                ++at;
            }
        __syncthreads();
        const uint32_t nout = min(total, static_cast<uint32_t>(kCandCap));
        for (uint32_t i = tid; i < nout; i += kTopkThreads)
            if (G + i < static_cast<uint32_t>(k)) o[G + i] = static_cast<int32_t>(opos[i]);
        return;
    }

    // ---- C: counts of this segment, offsets from the segments before it.
    // Each warp walks a contiguous part of the segment in blocks of 128 keys,
    // lane l taking keys 4l .. 4l+3 of a block with one 16-byte load (the
    // staged segment's storage is a multiple of 4 keys).
    const int wseg = ((m + kTopkWarps - 1) / kTopkWarps + 127) / 128 * 128;
    const int sb = warp * wseg, se = min(m, sb + wseg);
    auto load4 = [&](int i0, uint32_t (&u4)[4]) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i0 < se) v = *reinterpret_cast<const uint4*>(srow + i0);
        u4[0] = v.x;
        u4[1] = v.y;
        u4[2] = v.z;
        u4[3] = v.w;
    };
    uint32_t cg = 0, ce = 0;
    for (int base = sb; base < se; base += 128) {
        const int i0 = base + 4 * lane;
        uint32_t u4[4];
        load4(i0, u4);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool in = i0 + j < se;
            cg += (in && u4[j] > T) ? 1u : 0u;
            ce += (in && u4[j] == T) ? 1u : 0u;
        }
    }
    cg = __reduce_add_sync(0xffffffffu, cg);
    ce = __reduce_add_sync(0xffffffffu, ce);
    if (lane == 0) {
        S.wcnt[0][warp] = cg;
        S.wcnt[1][warp] = ce;
    }
    __syncthreads();
    // thread q > rank stores this segment's counts into CTA q's slot `rank`
    // (only the later segments offset by them)
    if (tid < kClusterCtas && tid > static_cast<int>(rank)) {
        uint32_t a = 0, b = 0;
        for (int w = 0; w < kTopkWarps; ++w) {
            a += S.wcnt[0][w];
            b += S.wcnt[1][w];
        }
        dsmem_st_u32(dsmem_addr(&CS.cnt_g[rank], tid), a);
        dsmem_st_u32(dsmem_addr(&CS.cnt_e[rank], tid), b);
    }
    // The last cluster barrier: every count is where it is needed, and every
    // remote load of this CTA's histograms and candidates came before it, so
    // from here each CTA touches only its own shared memory and may exit.
    cluster_sync_all();
    uint32_t G = 0, E = 0;
    for (uint32_t q = 0; q < rank; ++q) {
        G += CS.cnt_g[q];
        E += CS.cnt_e[q];
    }
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w)
        if (w < warp) {
            G += S.wcnt[0][w];
            E += S.wcnt[1][w];
        }
    const unsigned lt = (1u << lane) - 1u;
    for (int base = sb; base < se; base += 128) {
        const int i0 = base + 4 * lane;
        uint32_t u4[4];
        load4(i0, u4);
        bool gt[4], eq[4];
        unsigned bg[4], be[4];
        uint32_t g_before = G, e_before = E;  // keys > T and == T before this lane's first
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool in = i0 + j < se;
            gt[j] = in && u4[j] > T;
            eq[j] = in && u4[j] == T;
            bg[j] = __ballot_sync(0xffffffffu, gt[j]);
            be[j] = __ballot_sync(0xffffffffu, eq[j]);
            g_before += __popc(bg[j] & lt);
            e_before += __popc(be[j] & lt);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t pos =
                gt[j] ? g_before + (e_before < krem ? e_before : krem) : g_before + e_before;
            if ((gt[j] || (eq[j] && e_before < krem)) && pos < static_cast<uint32_t>(k))
                o[pos] = s0 + i0 + j;
            g_before += gt[j] ? 1u : 0u;
            e_before += eq[j] ? 1u : 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            G += __popc(bg[j]);
            E += __popc(be[j]);
        }
    }
}

static int launch_topk_cluster(ic_ctx* ctx, const float* scores, int64_t ld, int rows, int k,
                               int causal_base, const int32_t* row_len, int max_len,
                               int32_t* idx_out, int64_t ld_out, cudaStream_t stream,
                               uint32_t* hist) {
    const int seg_cap = ((max_len + kClusterCtas - 1) / kClusterCtas + 3) / 4 * 4;
    const int smem = (seg_cap + kCandCap) * 4;
    cudaError_t e = cudaFuncSetAttribute(k_topk_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaFuncSetAttribute(topk_cluster)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClusterCtas, rows, 1);
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterCtas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    unsigned int na = 1;
    add_pdl_attr(ctx, attr, na);
    cfg.attrs = attr;
    cfg.numAttrs = na;
    LaunchScope ls(ctx, IC_K_TOPK, stream);
    cudaLaunchKernelEx(&cfg, k_topk_cluster, scores, static_cast<long long>(ld), k, row_len,
                       max_len, causal_base, idx_out, static_cast<long long>(ld_out), seg_cap,
                       hist, ctx->dev_err);
    e = ls.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "topk_cluster launch");
    return IC_OK;
}

// one launch of the row kernel in the given shape (threads, candidate slots,
// and the CTAs per SM it is compiled for, 0 leaving the register count to
// the compiler), bcap the bitmap's keys
template <int THREADS, int CAND, int MINB>
static int launch_topk_rows(ic_ctx* ctx, const float* scores, int64_t ld, int rows, int k,
                            int causal_base, const int32_t* row_len, int max_len,
                            int32_t* idx_out, int64_t ld_out, int bcap, cudaStream_t stream) {
    static PerDeviceOnce attr_once;
    cudaError_t ea = attr_once.run(ctx->device, [] {
        return cudaFuncSetAttribute(k_topk<THREADS, CAND, MINB>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    CAND * 4 + kBitmapCap / 8);
    });
    if (ea != cudaSuccess) return cuda_fail(ctx, ea, "cudaFuncSetAttribute(topk)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rows, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = CAND * 4 + bcap / 8;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    unsigned int na = 0;
    add_pdl_attr(ctx, attr, na);
    cfg.attrs = attr;
    cfg.numAttrs = na;
    LaunchScope ls(ctx, IC_K_TOPK, stream);
    cudaLaunchKernelEx(&cfg, k_topk<THREADS, CAND, MINB>, scores, static_cast<long long>(ld), k,
                       causal_base, row_len, max_len, idx_out, static_cast<long long>(ld_out), bcap);
    cudaError_t e = ls.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "topk launch");
    return IC_OK;
}

bool topk_uses_cluster(const ic_ctx* ctx, int rows, bool has_row_len, int max_len) {
    // few long rows (decode): a cluster of CTAs per row keeps many SMs busy
    return has_row_len && rows > 0 &&
           static_cast<long long>(rows) * kClusterCtas <= 4LL * ctx->num_sms && max_len > 16384 &&
           max_len <= kClusterCtas * 45000;
}

int launch_topk(ic_ctx* ctx, const float* scores, int64_t ld, int rows, int k, int causal_base,
                const int32_t* row_len, int max_len, int32_t* idx_out, int64_t ld_out,
                cudaStream_t stream, uint32_t* hist) {
    if (rows <= 0) return IC_OK;
    if (topk_uses_cluster(ctx, rows, row_len != nullptr, max_len))
        return launch_topk_cluster(ctx, scores, ld, rows, k, causal_base, row_len, max_len, idx_out,
                                   ld_out, stream, hist);
    if (hist != nullptr)
        return fail(ctx, IC_ERR_INVALID_ARG, "topk: a histogram is only used by the cluster form");
    // causal row r has n = causal_base + r + 1 keys; rows longer than the
    // bitmap holds take the general path
    const long long nmax = row_len ? max_len : static_cast<long long>(causal_base) + rows;
    const int bcap = static_cast<int>(((nmax < kBitmapCap ? nmax : kBitmapCap) + 127) / 128 * 128);
    if (nmax <= kShortRow)
        return launch_topk_rows<256, 2048, 8>(ctx, scores, ld, rows, k, causal_base, row_len,
                                              max_len, idx_out, ld_out, bcap, stream);
    return launch_topk_rows<512, 4096, 0>(ctx, scores, ld, rows, k, causal_base, row_len, max_len,
                                          idx_out, ld_out, bcap, stream);
}

}  // namespace ic
