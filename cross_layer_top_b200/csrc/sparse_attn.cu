// Sparse MQA attention over gathered K/V rows:
//   o[r,h,:] = sum_{s in T_r} softmax_s(scale * Q[r,h,:].K[s,:]) V[s,:]
// ("IndexCache：跨层复用稀疏索引，以及它为什么能被训练", §3: each layer keeps
// its own Q/K/V and attends at the shared positions T_t; "IndexCache:
// Accelerating Sparse Attention via Cross-Layer Index Reuse", Figure 2 step
// SPARSEATTN).  One K/V head is shared by all Hq <= 16 query heads.
//
// Design: one CTA per (query row, key split): 3 warps and four CTAs per SM
// for whole rows (prefill), 4 warps and two CTAs per SM for split rows.
// The 16 query heads form the M = 16 rows of mma.m16n8k16 tiles, so one
// gathered K/V row serves every head.  Each warp owns chunks of 16 index
// slots and a 2-deep ring: lane l always copies the same 16-byte piece
// (l mod d/8) of its rows with cp.async (zero-filled for masked slots),
// XOR-swizzled by row so ldmatrix is conflict-free, while the warp computes
// an earlier chunk: S = Q K^T, an online softmax in the
// base-2 domain with the scale folded in and a lazy rescale (the running
// reference only moves when a logit exceeds it by 2^8, so O is rarely
// rescaled), and O += P V.  Slots holding -1 (or an out-of-range index,
// which is also latched as an error) are masked and gather zeros; the
// chunks after the last valid slot are skipped.  The warps' (m, l, O)
// merge through shared memory; one split writes bf16 output; with several
// splits (decode) the row's CTAs form a thread-block cluster and merge
// through distributed shared memory (each CTA owns a share of the heads and
// receives the other CTAs' partials of them in a receive area of its own,
// which leaves room for two such CTAs per SM).  A decode stack may pass the
// next layer's K/V (an S layer gathers at the same slots): its rows are then
// prefetched into L2 once this CTA's own gather is done.
#include "ic_device.cuh"
#include "ic_internal.h"

// Warps per CTA of the split (decode) and the row (prefill) kernel, and the
// gather-ring depth (compile-time tuning knobs).
#ifndef IC_ATTN_WARPS
#define IC_ATTN_WARPS 4
#endif
#ifndef IC_ATTN_ROW_WARPS
#define IC_ATTN_ROW_WARPS 3
#endif
#ifndef IC_ATTN_STAGES
#define IC_ATTN_STAGES 2
#endif

namespace ic {

// Split rows: rows of the receive area, >= nsplit * ceil(16 / nsplit) for
// every nsplit from 2 to 8 (at most 21, for nsplit = 7)
constexpr int kRecvRows = 24;

template <int D, int W>
struct AttnShape {
    static constexpr int WARPS = W;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int CH = 16;  // index slots per warp chunk
    static constexpr int STAGES = IC_ATTN_STAGES;
    static constexpr int ROWB = D * 2;
    static constexpr int ROWP = ROWB;  // row pitch; 16-byte pieces XOR-swizzled by row
    static constexpr int STAGE_BYTES = 2 * CH * ROWP;  // K rows then V rows
    static constexpr int WARP_BYTES = STAGES * STAGE_BYTES;
    static constexpr int Q_BYTES = 16 * ROWP;
    static constexpr int MAXK = 2048;
    static constexpr int OFF_IDX = 0;
    static constexpr int OFF_ST = OFF_IDX + MAXK * 4;
    // Q is staged in the last warp's second ring buffer, followed by the
    // CTA's last-valid-slot word: every warp reads both before any gather
    // fills that buffer
    static constexpr int OFF_Q = OFF_ST + (WARPS - 1) * WARP_BYTES + STAGE_BYTES;
    static constexpr int OFF_LAST = OFF_Q + Q_BYTES;
    // split rows (at most MAXK / 2 slots each) stage Q in the second half of
    // the slot area instead, so their first gathers need not wait for it
    static constexpr int OFF_Q_SPLIT = OFF_IDX + MAXK * 2;
    static_assert(Q_BYTES <= MAXK * 2, "Q fits half the slot area");
    static constexpr int SMEM = OFF_ST + WARPS * WARP_BYTES;
    // resident CTAs per SM (228 KB of shared memory, 1 KB reserved per CTA):
    // several CTAs keep several rows' prologues and merges in flight (three
    // 4-warp CTAs, or four 3-warp CTAs for the row kernel)
    static constexpr int CTAS_FIT = 233472 / (SMEM + 1024);
    static constexpr int CTAS_PER_SM = CTAS_FIT < 4 ? CTAS_FIT : 4;
    static_assert(CTAS_PER_SM >= 2, "shared memory per CTA");
    // split rows: a receive area of its own past the ring, for the cluster
    // merge ([kRecvRows][D] partial O, then [kRecvRows][2] M, L)
    static constexpr int OFF_RECV = SMEM;
    static constexpr int SMEM_SPLIT = OFF_RECV + (kRecvRows * D + kRecvRows * 2) * 4;
    static constexpr int CTAS_SPLIT = 233472 / (SMEM_SPLIT + 1024) < 3 ? 233472 / (SMEM_SPLIT + 1024) : 3;
    static_assert(Q_BYTES + 4 <= STAGE_BYTES && STAGES >= 2, "Q and the last-slot word live in a second ring buffer");
    // per-warp O and (m, l), then the per-head factors, M and L
    // per-warp partial O rows are OS = D + 8 floats apart (OS = 8 mod 32 banks):
    // a warp's float2 fragment stores then take the minimal two wavefronts
    static constexpr int OS = D + 8;
    static constexpr int MERGE_BYTES = WARPS * (16 * OS + 32) * 4 + (WARPS * 16 + 32) * 4;
    static_assert(MERGE_BYTES <= WARPS * WARP_BYTES, "merge buffer must fit in the stages");
};

// byte offset of 16-byte piece c of row `row` in a [rows][d] bf16 tile whose
// pieces are XOR-swizzled by (row mod 8): ldmatrix reads 8 rows of one piece
// column from 8 different bank groups
// CTAs of one split row's cluster, at most: the portable cluster size (on
// back-to-back decode layers 8-CTA clusters schedule better than 16 or 4)
constexpr int kMaxClusterSplits = 8;
// receive rows an owner needs for nsplit splits of 16 heads: nsplit * ceil(16 / nsplit)
constexpr int recv_rows_for(int n) {
    return n <= 1 ? 16 : (n * ((16 + n - 1) / n) > recv_rows_for(n - 1) ? n * ((16 + n - 1) / n)
                                                                          : recv_rows_for(n - 1));
}
static_assert(recv_rows_for(kMaxClusterSplits) <= kRecvRows, "receive area holds every split");

template <int D>
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return static_cast<uint32_t>(row * (D * 2) + ((c ^ (row & 7)) << 4));
}

// One chunk of CH = 16 gathered slots (K rows at kb, V rows at vb, swizzled)
// folded into a warp's running state: S = Q K^T on the tensor cores, slots
// whose cmask bit is clear set to -inf, an online softmax in the base-2
// domain with a lazy rescale (the reference m moves only when a logit passes
// it by 2^kRescaleThreshold), then O += P V.  Rows g = lane/4 and g + 8 of
// the 16 heads; m, l per row (l is this lane's partial sum).
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
__device__ __forceinline__ void attn_chunk(uint32_t kb, uint32_t vb, uint32_t cmask,
                                           const uint32_t (&qa)[D / 16][4], float (&o)[D / 8][4],
                                           float& m0, float& m1, float& l0, float& l1,
                                           float scale_log2, int lane) {
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    // two accumulator chains per 8-key tile (the even and the odd 16-wide
    // steps, added at the end), so each chain of dependent MMAs is half as
    // long (measured: 1.000 -> 0.981 ms per prefill layer)
    float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int m = lane >> 3;
        const int key = (m >> 1) * 8 + (lane & 7);
        const int c = 2 * kk + (m & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz<D>(key, c), b0, b1, b2, b3);
        float(&t0)[4] = (kk & 1) ? s2[0] : s[0];
        float(&t1)[4] = (kk & 1) ? s2[1] : s[1];
        mma_bf16_16816(t0, qa[kk], b0, b1);
        mma_bf16_16816(t1, qa[kk], b2, b3);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
    if (cmask != 0xffffu) {  // warp-uniform: only chunks with masked slots
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = nt * 8 + 2 * (lane & 3) + (e & 1);
                if (!((cmask >> col) & 1u)) s[nt][e] = -INFINITY;
            }
    }
    float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    mx0 *= scale_log2;  // scale > 0 keeps the order
    mx1 *= scale_log2;
    // lazy rescale: move the reference only when a logit passes it by 2^8
    if (mx0 > m0 + kRescaleThreshold) {
        const float a = ex2_approx(m0 - mx0);  // 0 while nothing was seen
        l0 *= a;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            o[i][0] *= a;
            o[i][1] *= a;
        }
        m0 = mx0;
    }
    if (mx1 > m1 + kRescaleThreshold) {
        const float a = ex2_approx(m1 - mx1);
        l1 *= a;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            o[i][2] *= a;
            o[i][3] *= a;
        }
        m1 = mx1;
    }
    const float n0 = m0 == -INFINITY ? 0.f : -m0;
    const float n1 = m1 == -INFINITY ? 0.f : -m1;
    float p[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        p[nt][0] = ex2_approx(fmaf(s[nt][0], scale_log2, n0));
        p[nt][1] = ex2_approx(fmaf(s[nt][1], scale_log2, n0));
        p[nt][2] = ex2_approx(fmaf(s[nt][2], scale_log2, n1));
        p[nt][3] = ex2_approx(fmaf(s[nt][3], scale_log2, n1));
    }
    l0 += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
    l1 += (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
    uint32_t pa[4];
    pa[0] = pack_bf16x2(p[0][0], p[0][1]);
    pa[1] = pack_bf16x2(p[0][2], p[0][3]);
    pa[2] = pack_bf16x2(p[1][0], p[1][1]);
    pa[3] = pack_bf16x2(p[1][2], p[1][3]);
#pragma unroll
    for (int dn = 0; dn < D / 16; ++dn) {
        const int m = lane >> 3;
        const int key = (m & 1) * 8 + (lane & 7);
        const int c = 2 * dn + (m >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz<D>(key, c), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * dn], pa, b0, b1);
        mma_bf16_16816(o[2 * dn + 1], pa, b2, b3);
    }
}

// SPLIT: rows split across a cluster of CTAs (few rows, decode); otherwise
// one CTA per row, and the cluster merge is not compiled in.
// the shape of the split (decode) and of the row (prefill) kernel
template <int D, bool SPLIT>
using AttnShapeOf = AttnShape<D, SPLIT ? IC_ATTN_WARPS : IC_ATTN_ROW_WARPS>;

template <int D, bool SPLIT>
__global__ void __launch_bounds__(AttnShapeOf<D, SPLIT>::THREADS,
                                  SPLIT ? AttnShapeOf<D, SPLIT>::CTAS_SPLIT
                                        : AttnShapeOf<D, SPLIT>::CTAS_PER_SM)
    k_sparse_attn(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                  const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ idx, int Hq,
                  int k, int rows_per_seq, long long kv_seq_stride, int kv_len, float scale_log2,
                  int nsplit, int kps, int pf_ahead, int vec_idx, int pdl,
                  const __nv_bfloat16* __restrict__ nK, const __nv_bfloat16* __restrict__ nV,
                  __nv_bfloat16* __restrict__ out,
                  int* __restrict__ err) {
    using S = AttnShapeOf<D, SPLIT>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int r = blockIdx.x, split = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slot0 = split * kps;
    const int nk = max(0, min(k, slot0 + kps) - slot0);
    int32_t* sIdx = reinterpret_cast<int32_t*>(smem + S::OFF_IDX);
    int* s_last = reinterpret_cast<int*>(smem + S::OFF_LAST);
    const uint32_t sQ = smem_u32(smem + (SPLIT ? S::OFF_Q_SPLIT : S::OFF_Q));
    const long long seq = rows_per_seq > 0 ? r / rows_per_seq : 0;
    const __nv_bfloat16* Kb = K + seq * kv_seq_stride;
    const __nv_bfloat16* Vb = V + seq * kv_seq_stride;

    // rows run about one wave of CTAs apart: warm L2 with the index and
    // query rows of the row one wave ahead, so whichever CTA takes it does not
    // start on an HBM round trip
    if (!SPLIT && pf_ahead > 0 && r + pf_ahead < gridDim.x) {
        const int rr = r + pf_ahead;
        const char* pidx = reinterpret_cast<const char*>(idx + static_cast<long long>(rr) * k);
        const char* pq = reinterpret_cast<const char*>(Q + static_cast<long long>(rr) * Hq * D);
        const int idx_lines = (k * 4 + 127) / 128, q_lines = (Hq * D * 2 + 127) / 128;
        if (tid < idx_lines)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(pidx + tid * 128));
        else if (tid < idx_lines + q_lines)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(pq + (tid - idx_lines) * 128));
    }
    // a split row's CTAs arrive on the cluster barrier at once and wait on it
    // only before their first remote store, so that every CTA of the cluster
    // is known to be running by then
    if constexpr (SPLIT) cluster_arrive_relaxed();
    if (tid == 0) *s_last = -1;
    __syncthreads();
    // the query heads go to shared memory by cp.async, in flight while the
    // index slots load (zeros for heads past Hq)
    const __nv_bfloat16* qrow = Q + static_cast<long long>(r) * Hq * D;
    auto stage_q = [&]() {
        for (int p = tid; p < 16 * (D / 8); p += S::THREADS) {
            const int h = p / (D / 8), c = p % (D / 8);
            const bool ok = h < Hq;
            cp_async16(sQ + swz<D>(h, c), ok ? qrow + h * D + c * 8 : qrow, ok);
        }
        cp_async_commit();
    };
    // as a programmatic dependent (pdl 1): nothing is read before the previous
    // kernel completes; pdl 2 (an S layer) waits below, after the index slots
    if (pdl != 2) {
        griddep_wait();
        stage_q();
    }
    // index slots of this split (validated), the last valid slot, the query heads
    const int32_t* irow = idx + static_cast<long long>(r) * k + slot0;
    bool bad = false;
    int last = -1;
    const int nk_pad = (nk + S::CH - 1) / S::CH * S::CH;  // whole chunks, padded with -1
    auto take = [&](int i, int v) {  // validate slot i; -1 (masked) for a bad index
        if (v < -1 || v >= kv_len) {
            bad = true;
            v = -1;
        }
        if (v >= 0) last = i;
        return v;
    };
    if (vec_idx) {  // 16-byte aligned slot rows, nk a multiple of 4: four slots per load
        for (int i = 4 * tid; i < nk_pad; i += 4 * S::THREADS) {
            int4 v = make_int4(-1, -1, -1, -1);
            if (i < nk) v = __ldg(reinterpret_cast<const int4*>(irow + i));
            v.x = take(i, v.x);
            v.y = take(i + 1, v.y);
            v.z = take(i + 2, v.z);
            v.w = take(i + 3, v.w);
            *reinterpret_cast<int4*>(sIdx + i) = v;
        }
    } else {
        for (int i = tid; i < nk_pad; i += S::THREADS) sIdx[i] = take(i, i < nk ? irow[i] : -1);
    }
    if (bad) atomicCAS(err, 0, kDevBadIndex);
    last = __reduce_max_sync(0xffffffffu, last);
    if (lane == 0 && last >= 0) atomicMax(s_last, last);
    // warm L2 with the K and V rows of a layer (base pointers kb, vb of this
    // row's sequence) at this split's first n staged slots
    auto prefetch_rows = [&](const __nv_bfloat16* kb, const __nv_bfloat16* vb, int n) {
        constexpr int LPR = (D * 2 + 127) / 128;  // 128-byte lines per row
        for (int t = tid; t < n * 2 * LPR; t += S::THREADS) {
            const int slot = t / (2 * LPR), part = t - slot * (2 * LPR);
            const int v = sIdx[slot];
            if (v >= 0) {
                const char* row = reinterpret_cast<const char*>(part < LPR ? kb : vb) +
                                  static_cast<long long>(v) * D * 2 + (part % LPR) * 128;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(row));
            }
        }
    };
    if (pdl == 2) {
        // An S layer's index slots and its cached K/V rows are not written by
        // the previous kernel: warm L2 with the rows this split will gather,
        // then wait for that kernel before reading the query heads (and, in
        // the main loop, the rows themselves, the newest one included).
        __syncthreads();  // every slot is staged
        prefetch_rows(Kb, Vb, nk);
        griddep_wait();
        stage_q();
    }
    griddep_launch_dependents();
    if constexpr (!SPLIT) cp_async_wait<0>();  // Q, in a ring buffer, is read before any gather
    __syncthreads();
    const int nk_eff = *s_last + 1;  // slots after the last valid one hold nothing

    uint32_t qa[D / 16][4];
    auto load_q = [&]() {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int m = lane >> 3;
            const int row = (m & 1) * 8 + (lane & 7);
            const int c = 2 * kk + (m >> 1);
            ldsm_x4(sQ + swz<D>(row, c), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
        }
    };
    if constexpr (!SPLIT) load_q();
    // every warp holds Q (row kernel) and has read the last-slot word, which
    // lies in a ring buffer: the gathers may now fill the ring
    __syncthreads();

    const uint32_t wst = smem_u32(smem + S::OFF_ST + warp * S::WARP_BYTES);
    const int nch = (nk_eff + S::CH - 1) / S::CH;
    const int my_n = nch > warp ? (nch - warp + S::WARPS - 1) / S::WARPS : 0;

    // lane l copies piece (l % PPR) of rows l / PPR, + RPI, ... of K and V.
    // Its destination in a stage, swz(prow + i*RPI, piece), is computed
    // where used: prow < RPI and RPI is a power of two, so
    // (prow + i*RPI) & 7 = prow ^ ((i*RPI) & 7) and the swizzled piece is
    // (piece ^ prow) ^ ((i*RPI) & 7), one XOR with a constant per copy
    // (registers are what bound the CTAs per SM here).
    constexpr int PPR = D / 8;        // 16-byte pieces per row
    constexpr int RPI = 32 / PPR;     // rows per warp instruction
    constexpr int NI = S::CH / RPI;   // copy instructions per lane per tensor
    const int piece = lane % PPR, prow = lane / PPR;
    const uint32_t dbase = static_cast<uint32_t>(prow * S::ROWB);
    const uint32_t dpiece = static_cast<uint32_t>((piece ^ prow) << 4);
    auto dst_off = [&](int i) {
        return dbase + static_cast<uint32_t>(i * RPI * S::ROWB) +
               (dpiece ^ static_cast<uint32_t>(((i * RPI) & 7) << 4));
    };
    const char* Kc = reinterpret_cast<const char*>(Kb) + piece * 16;
    const char* Vc = reinterpret_cast<const char*>(Vb) + piece * 16;
    static_assert(RPI == 2 || RPI == 4, "slot selection below");
    // This lane's NI slots of chunk j (its rows prow + i * RPI), read as the
    // chunk's CH / 4 16-byte broadcast loads and reduced to the NI it uses
    // (chunks past the warp's last read chunk 0's, unused).
    auto load_slots = [&](int j, int (&sl)[NI]) {
        const int c0 = (warp + (j < my_n ? j : 0) * S::WARPS) * S::CH;
        int4 sv[S::CH / 4];
#pragma unroll
        for (int q = 0; q < S::CH / 4; ++q) sv[q] = *reinterpret_cast<const int4*>(sIdx + c0 + 4 * q);
#pragma unroll
        for (int i = 0; i < NI; ++i) {  // row prow + i*RPI: vector (i*RPI)/4, element prow + (i*RPI)%4
            const int4 v = sv[(i * RPI) / 4];
            const bool b0 = prow & 1;
            const bool b1 = RPI == 2 ? ((i * RPI) & 2) != 0 : (prow & 2) != 0;
            sl[i] = b1 ? (b0 ? v.w : v.z) : (b0 ? v.y : v.x);
        }
    };
    // gather chunk j's K and V rows into its stage
    auto issue_with = [&](int j, const int (&sl)[NI]) {
        if (j < my_n) {
            const uint32_t kdst = wst + (j % S::STAGES) * S::STAGE_BYTES;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int sidx = sl[i];
                const bool ok = sidx >= 0;
                const uint32_t off = static_cast<uint32_t>(ok ? sidx : 0) * S::ROWB;
                const uint32_t d = kdst + dst_off(i);
                cp_async16(d, Kc + off, ok);
                cp_async16(d + S::CH * S::ROWP, Vc + off, ok);
            }
        }
        cp_async_commit();
    };
    auto issue = [&](int j) {
        int sl[NI];
        load_slots(j, sl);
        issue_with(j, sl);
    };

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    // running references (log2 domain, scale folded in) and partial sums,
    // rows g = lane/4 and g + 8
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    // every stage starts filled; the stage of chunk j is refilled (chunk
    // j + STAGES) as soon as chunk j has been consumed
#pragma unroll
    for (int j = 0; j < S::STAGES; ++j) issue(j);
    if constexpr (SPLIT) {
        // split rows stage Q outside the ring, so the first gathers went out
        // before it landed; its cp.async group is older than theirs
        cp_async_wait<S::STAGES>();
        __syncthreads();
        load_q();
    }
    for (int j = 0; j < my_n; ++j) {
        const int st = j % S::STAGES;
        cp_async_wait<S::STAGES - 1>();  // chunk j has landed
        __syncwarp();
        const uint32_t kb = wst + st * S::STAGE_BYTES;
        const uint32_t vb = kb + S::CH * S::ROWP;
        const int c0 = (warp + j * S::WARPS) * S::CH;
        const uint32_t cmask = __ballot_sync(0xffffffffu, sIdx[c0 + (lane & 15)] >= 0) & 0xffffu;

        // the slots of the gather that refills this stage are read before the
        // compute, so their latency is not paid between chunks
        int nsl[NI];
        load_slots(j + S::STAGES, nsl);
        attn_chunk<D>(kb, vb, cmask, qa, o, m0, m1, l0, l1, scale_log2, lane);
        __syncwarp();                    // every lane is done reading stage st
        issue_with(j + S::STAGES, nsl);  // refill it
    }
    cp_async_wait<0>();
    // the next layer (an S layer) gathers its own K/V at these same slots:
    // its rows are fetched into L2 while this row merges
    if (nK != nullptr) prefetch_rows(nK + seq * kv_seq_stride, nV + seq * kv_seq_stride, nk_eff);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    __syncthreads();  // every warp is done with its stages: reuse them for the merge

    float* mO = reinterpret_cast<float*>(smem + S::OFF_ST);  // [WARPS][16][OS]
    float* mML = mO + S::WARPS * 16 * S::OS;                 // [WARPS][32]: m[16], l[16]
    {
        const int g = lane >> 2, cc = 2 * (lane & 3);
        float* ow = mO + warp * 16 * S::OS;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            *reinterpret_cast<float2*>(ow + g * S::OS + i * 8 + cc) = make_float2(o[i][0], o[i][1]);
            *reinterpret_cast<float2*>(ow + (g + 8) * S::OS + i * 8 + cc) =
                make_float2(o[i][2], o[i][3]);
        }
        if ((lane & 3) == 0) {
            mML[warp * 32 + g] = m0;
            mML[warp * 32 + g + 8] = m1;
            mML[warp * 32 + 16 + g] = l0;
            mML[warp * 32 + 16 + g + 8] = l1;
        }
    }
    __syncthreads();
    // combine the warps: per head M = max_w m_w, factors f_w = 2^(m_w - M),
    // L = sum_w l_w f_w (computed once per head), then o = sum_w O_w f_w
    // over float4 columns
    float* sF = mML + S::WARPS * 32;  // [WARPS][16] factors, then M[16], L[16]
    if (tid < 16) {
        const int h = tid;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < S::WARPS; ++w) M = fmaxf(M, mML[w * 32 + h]);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < S::WARPS; ++w) {
            const float f = M == -INFINITY ? 0.f : ex2_approx(mML[w * 32 + h] - M);
            sF[w * 16 + h] = f;
            L += mML[w * 32 + 16 + h] * f;
        }
        sF[S::WARPS * 16 + h] = M;
        sF[S::WARPS * 16 + 16 + h] = L;
    }
    __syncthreads();
    // this CTA's combined o[h][d4..d4+3] = sum_w O_w f_w (relative to its M[h])
    auto combine = [&](int h, int d4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < S::WARPS; ++w) {
            const float f = sF[w * 16 + h];
            const float4 v = *reinterpret_cast<const float4*>(mO + (w * 16 + h) * S::OS + d4);
            acc.x = fmaf(v.x, f, acc.x);
            acc.y = fmaf(v.y, f, acc.y);
            acc.z = fmaf(v.z, f, acc.z);
            acc.w = fmaf(v.w, f, acc.w);
        }
        return acc;
    };
    if (!SPLIT) {
        for (int e4 = tid; e4 < Hq * (D / 4); e4 += S::THREADS) {
            const int h = e4 / (D / 4), d4 = (e4 % (D / 4)) * 4;
            const float4 acc = combine(h, d4);
            const float L = sF[S::WARPS * 16 + 16 + h];
            const float iv = L > 0.f ? 1.f / L : 0.f;
            __nv_bfloat16* op = out + (static_cast<long long>(r) * Hq + h) * D + d4;
            *reinterpret_cast<uint2*>(op) = make_uint2(pack_bf16x2(acc.x * iv, acc.y * iv),
                                                       pack_bf16x2(acc.z * iv, acc.w * iv));
        }
        return;
    }

    // Split rows: the row's nsplit CTAs form one thread-block cluster.  CTA q
    // owns heads [q*hpc, (q+1)*hpc); every CTA stores its combined partial of
    // those heads (O relative to its M, and M, L) into the owner's receive
    // area with distributed-shared-memory stores, and each owner merges
    //   out = sum_q O_q 2^(M_q - M) / sum_q L_q 2^(M_q - M),  M = max_q M_q.
    // The receive area is used by nothing else, so a CTA stores as soon as
    // its own partial is ready; one cluster barrier (arrive with release,
    // wait with acquire) then makes every store visible to its owner.  After
    // it each CTA reads only its own shared memory, so it may exit when done.
    cluster_wait_acquire();  // every CTA of the cluster is running
    const int hpc = (16 + nsplit - 1) / nsplit;  // heads per owner
    const uint32_t q = cluster_rank();
    float* rO = reinterpret_cast<float*>(smem + S::OFF_RECV);  // [nsplit][hpc][D] received O
    float* rML = rO + kRecvRows * D;                           // [nsplit][hpc][2] received M, L
    for (int e4 = tid; e4 < 16 * (D / 4); e4 += S::THREADS) {
        const int h = e4 / (D / 4), d4 = (e4 % (D / 4)) * 4;
        const int owner = h / hpc, hl = h - owner * hpc;
        dsmem_st_f4(dsmem_addr(rO + (q * hpc + hl) * D + d4, owner), combine(h, d4));
    }
    if (tid < 16) {
        const int h = tid, owner = h / hpc, hl = h - owner * hpc;
        dsmem_st_f32(dsmem_addr(rML + (q * hpc + hl) * 2, owner), sF[S::WARPS * 16 + h]);
        dsmem_st_f32(dsmem_addr(rML + (q * hpc + hl) * 2 + 1, owner), sF[S::WARPS * 16 + 16 + h]);
    }
    cluster_arrive_release();
    cluster_wait_acquire();
    for (int e4 = tid; e4 < hpc * (D / 4); e4 += S::THREADS) {
        const int hl = e4 / (D / 4), d4 = (e4 % (D / 4)) * 4;
        const int h = static_cast<int>(q) * hpc + hl;
        if (h >= Hq) continue;
        float M = -INFINITY;
        for (int p = 0; p < nsplit; ++p) M = fmaxf(M, rML[(p * hpc + hl) * 2]);
        float L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int p = 0; p < nsplit; ++p) {
            const float f = M == -INFINITY ? 0.f : ex2_approx(rML[(p * hpc + hl) * 2] - M);
            L += rML[(p * hpc + hl) * 2 + 1] * f;
            const float4 v = *reinterpret_cast<const float4*>(rO + (p * hpc + hl) * D + d4);
            acc.x = fmaf(v.x, f, acc.x);
            acc.y = fmaf(v.y, f, acc.y);
            acc.z = fmaf(v.z, f, acc.z);
            acc.w = fmaf(v.w, f, acc.w);
        }
        const float iv = L > 0.f ? 1.f / L : 0.f;
        __nv_bfloat16* op = out + (static_cast<long long>(r) * Hq + h) * D + d4;
        *reinterpret_cast<uint2*>(op) = make_uint2(pack_bf16x2(acc.x * iv, acc.y * iv),
                                                   pack_bf16x2(acc.z * iv, acc.w * iv));
    }
}

template <int D>
static int launch_attn_t(ic_ctx* ctx, const void* Q, const void* K, const void* V,
                         const int32_t* idx, int rows, int Hq, int k, int rows_per_seq,
                         int64_t kv_seq_stride, int kv_len, float scale, void* out,
                         cudaStream_t stream) {
    using SR = AttnShapeOf<D, false>;  // the row kernel
    using SS = AttnShapeOf<D, true>;   // the split kernel
    static PerDeviceOnce attr_once;
    cudaError_t ea = attr_once.run(ctx->device, [] {
        cudaError_t e = cudaFuncSetAttribute(k_sparse_attn<D, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, SR::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_sparse_attn<D, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, SS::SMEM_SPLIT);
        return e;
    });
    if (ea != cudaSuccess) return cuda_fail(ctx, ea, "cudaFuncSetAttribute(sparse_attn)");
    // Split the index slots across CTAs when there are too few rows to fill
    // the GPU (decode): about one wave of resident CTAs, whole chunks per
    // split, at most kMaxClusterSplits.  A split row's CTAs form one cluster
    // (they merge through distributed shared memory); the split count is
    // lowered until every row's cluster can be resident at once (a cluster
    // waiting for a second wave would double the kernel's time).
    // resident clusters per device and cluster size (0: not yet asked)
    static std::atomic<int> active[kMaxDevices][kMaxClusterSplits + 1] = {};
    const int dev = ctx->device >= 0 && ctx->device < kMaxDevices ? ctx->device : 0;
    auto resident_clusters = [&](int cs) -> int {
        int n = active[dev][cs].load(std::memory_order_relaxed);
        if (n == 0) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(1, cs, 1);
            q.blockDim = dim3(SS::THREADS, 1, 1);
            q.dynamicSmemBytes = SS::SMEM_SPLIT;
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = 1;
            qa[0].val.clusterDim.y = cs;
            qa[0].val.clusterDim.z = 1;
            q.attrs = qa;
            q.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, k_sparse_attn<D, true>, &q) != cudaSuccess) n = -1;
            cudaGetLastError();  // a refused query leaves no error behind
            active[dev][cs].store(n, std::memory_order_relaxed);
        }
        return n;
    };
    int nsplit = 1;
    const int target = SR::CTAS_PER_SM * ctx->num_sms;
    if (rows < target) {
        nsplit = target / rows;
        const int max_split = (k + SS::CH - 1) / SS::CH;
        if (nsplit > max_split) nsplit = max_split;
        if (nsplit > kMaxClusterSplits) nsplit = kMaxClusterSplits;
        while (nsplit > 1 && resident_clusters(nsplit) < rows) --nsplit;
        if (nsplit < 1) nsplit = 1;
    }
    int kps = (k + nsplit - 1) / nsplit;
    kps = (kps + SS::CH - 1) / SS::CH * SS::CH;
    nsplit = (k + kps - 1) / kps;
    const float scale_log2 = scale * 1.4426950408889634f;
    // slot rows start 16-byte aligned when idx does and k, kps are multiples of 4
    const int vec_idx = (reinterpret_cast<uintptr_t>(idx) & 15) == 0 && k % 4 == 0 && kps % 4 == 0;
    LaunchScope ls(ctx, IC_K_ATTN, stream);
    const auto* Qp = static_cast<const __nv_bfloat16*>(Q);
    const auto* Kp = static_cast<const __nv_bfloat16*>(K);
    const auto* Vp = static_cast<const __nv_bfloat16*>(V);
    auto* op = static_cast<__nv_bfloat16*>(out);
    // the next layer's K/V, to prefetch at these slots (both or neither)
    const auto* pfK = ctx->pf_V ? static_cast<const __nv_bfloat16*>(ctx->pf_K) : nullptr;
    const auto* pfV = pfK ? static_cast<const __nv_bfloat16*>(ctx->pf_V) : nullptr;
    const long long kvs = static_cast<long long>(kv_seq_stride);
    // a split row's slots share the slot area with Q (k <= 2048 over >= 2 splits)
    if (nsplit > 1 && kps > SS::MAXK / 2)
        return fail(ctx, IC_ERR_UNSUPPORTED, "sparse_attn: %d slots per split", kps);
    if (nsplit == 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(rows, 1, 1);
        cfg.blockDim = dim3(SR::THREADS, 1, 1);
        cfg.dynamicSmemBytes = SR::SMEM;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        unsigned int na = 0;
        add_pdl_attr(ctx, attr, na);
        cfg.attrs = attr;
        cfg.numAttrs = na;
        cudaLaunchKernelEx(&cfg, k_sparse_attn<D, false>, Qp, Kp, Vp, idx, Hq, k, rows_per_seq, kvs,
                           kv_len, scale_log2, 1, kps, SR::CTAS_PER_SM * ctx->num_sms, vec_idx,
                           ctx->pdl, pfK, pfV, op, ctx->dev_err);
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(rows, nsplit, 1);
        cfg.blockDim = dim3(SS::THREADS, 1, 1);
        cfg.dynamicSmemBytes = SS::SMEM_SPLIT;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = nsplit;
        attr[0].val.clusterDim.z = 1;
        unsigned int na = 1;
        add_pdl_attr(ctx, attr, na);
        cfg.attrs = attr;
        cfg.numAttrs = na;
        cudaLaunchKernelEx(&cfg, k_sparse_attn<D, true>, Qp, Kp, Vp, idx, Hq, k, rows_per_seq, kvs, kv_len,
                           scale_log2, nsplit, kps, 0, vec_idx, ctx->pdl, pfK, pfV, op,
                           ctx->dev_err);
    }
    cudaError_t e = ls.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "sparse_attn launch");
    return IC_OK;
}

int launch_sparse_attn(ic_ctx* ctx, const void* Q, const void* K, const void* V,
                       const int32_t* idx, int rows, int Hq, int d, int k, int rows_per_seq,
                       int64_t kv_seq_stride, int kv_len, float scale, void* out,
                       cudaStream_t stream) {
    if (rows <= 0) return IC_OK;
    if (d == 128)
        return launch_attn_t<128>(ctx, Q, K, V, idx, rows, Hq, k, rows_per_seq, kv_seq_stride,
                                  kv_len, scale, out, stream);
    if (d == 64)
        return launch_attn_t<64>(ctx, Q, K, V, idx, rows, Hq, k, rows_per_seq, kv_seq_stride,
                                 kv_len, scale, out, stream);
    return fail(ctx, IC_ERR_UNSUPPORTED, "sparse_attn: d=%d not in {64,128}", d);
}

}  // namespace ic
