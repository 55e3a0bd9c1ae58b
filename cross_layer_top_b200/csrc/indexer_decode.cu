// Decode-step lightning-indexer scan over an FP8 indexer-key cache.
//
// For one new query token per sequence b and every cached candidate s:
//   I[b,s] = scale[b,s] * sum_j w[b,j] * ReLU(q[b,j,:] . e4m3(k8[b,s,:]))
// which equals the score of "IndexCache：跨层复用稀疏索引，以及它为什么能被训练"
// §2.1 on the dequantised key k[b,s,:] = e4m3(k8[b,s,:]) * scale[b,s],
// because scale > 0 commutes with ReLU.  The decode step scans the whole
// cache ("IndexCache：…", §10.1); the indexer runs in FP8 ("IndexCache:
// Accelerating Sparse Attention via Cross-Layer Index Reuse", §2.1).
//
// Design (sm_100a), one persistent CTA per SM, HBM-bound by construction.
// The e4m3 key tile goes from HBM to the tensor core untouched: TMA writes
// it in the 128-byte-swizzle K-major layout and UMMA kind::f8f6f4 reads it
// as the A operand.  The bf16 query is carried exactly by two e4m3 terms:
// with x = q * 2^s (2^s puts max|x| in [2^7, 2^8)), hi = e4m3(x) and
// lo = e4m3(x - hi) give hi + lo = x exactly for every |x| >= 2^-2 (the
// remainder x - hi is a multiple of x's bf16 ulp no larger than 8 ulps, so
// it has at most four significant bits), and within 2^-10 (2^-17 of max|x|)
// below that.  hi and lo are stacked as the 2 H_I rows of one B operand
// (an M = 128 UMMA costs the same for any N <= 64, so N = 2 H_I is free):
// D[s,j] = k_s . hi_j and D[s,H_I+j] = k_s . lo_j, added in the epilogue.
//  * warp 0 (TMA): streams key tiles (256 keys x 128 B, one tensor copy)
//    through a 5-deep ring; rows past the end of the cache read as zero and
//    are never stored;
//  * warps 4..7 (query): when the CTA's range enters a new sequence, read
//    its q, find 2^s and write hi / lo (double-buffered, swizzled);
//  * warp 1 (MMA): per tile, 4 UMMAs (M = 128 keys, N = 2 H_I, K = 32) for
//    each 128-key half into its own accumulator, fp32 in TMEM; one commit
//    per tile for the stage and one for the accumulator pair (the per-tile
//    fixed costs are what bound the issuer, so tiles are 256 keys);
//  * warps 8..15 (epilogue; warps 8..11 take the first half of each tile,
//    12..15 the second): the thread owning TMEM lane s adds hi and lo,
//    applies ReLU, the w weights, the head sum, 2^-s and the per-token
//    scale, and stores I[b,s].
// Each CTA scans a contiguous range of (sequence, key tile) pairs.  All
// waits are bounded.
// When asked (hist != NULL) the epilogue also counts the scores it stores
// per sequence into 2048 bins by the top 11 bits of their order key, the
// first radix digit of the top-k that follows: hist[b][bin] += count.  The
// counts of the CTA's first and last sequence gather in shared memory and
// go out with one atomic add per nonzero bin at the end; a sequence in
// between, which only this CTA touches, is counted straight into hist.
// hist must be zero before the launch (the top-k clears it after use).
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

template <int H_I>
struct DecodeShape {
    static constexpr int BM = 256;          // keys per tile (two UMMA halves of 128)
    static constexpr int DI = 128;          // d_I (bytes per e4m3 key row)
    static constexpr int A_BYTES = BM * DI; // one key tile
    static constexpr int A_HALF = 128 * DI;
    static constexpr int A_ST = 5;
    static constexpr int B_HALF = H_I * DI; // hi or lo: H_I rows of 128 e4m3
    static constexpr int B_BUF = 2 * B_HALF;
    static constexpr int ACC_COLS = 2 * H_I;  // hi heads, then lo heads
    static constexpr int TMEM_COLS = 512;
    static constexpr int NACC = TMEM_COLS / (2 * ACC_COLS);  // accumulator pairs (one per tile)
    // per-sequence ring (query warps -> epilogue): tag b, 2^-s, w[b,:] in fp32
    static constexpr int SEQ_RING = 8;
    static constexpr int SEQ_BYTES = 16 + 4 * H_I;
    static constexpr int W_BYTES = SEQ_RING * SEQ_BYTES;
    static constexpr int SC_RING = 8;       // scale prefetch depth (tiles)
    static constexpr int SC_BYTES = SC_RING * BM * 4;
    static constexpr int QRED_BYTES = 32;   // [2][4] warp maxima of |q|
    static constexpr int HIST_BYTES = 2 * kKeyBins * 4;  // first / last sequence's counts
    static constexpr int BAR_BYTES = 512;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + A_ST * A_BYTES;
    static constexpr int OFF_W = OFF_B + 2 * B_BUF;
    static constexpr int OFF_SC = OFF_W + W_BYTES;
    static constexpr int OFF_QRED = OFF_SC + SC_BYTES;
    static constexpr int OFF_HIST = OFF_QRED + QRED_BYTES;
    static constexpr int OFF_BAR = OFF_HIST + HIST_BYTES;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(NACC >= 2, "TMEM allocation");
    static_assert(OFF_B % 1024 == 0 && B_HALF % 1024 == 0, "swizzle atoms need 1024-B alignment");
};

// e4m3 pair <-> float pair.  The low byte is the first element.
__device__ __forceinline__ uint32_t e4m3x2_of(float first, float second) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
    return r;
}
__device__ __forceinline__ float2 float2_of_e4m3x2(uint32_t pair16) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<unsigned short>(pair16)));
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// The power of two 2^s that brings the largest |q| of a sequence (bf16 bit
// pattern M of its magnitude) into [2^7, 2^8), clamped to normal floats.
__device__ __forceinline__ int q_shift_of_max(uint32_t M) {
    const int e = static_cast<int>((M >> 7) & 0xFF) - 127;
    const int sh = M == 0 ? 0 : 7 - e;
    return sh > 126 ? 126 : (sh < -126 ? -126 : sh);
}
// Walks a CTA's contiguous range of (sequence b, key tile j) pairs in order,
// visiting only tiles that hold candidates (j * BM < seq_len[b]) and
// skipping a sequence's empty tail in one step.  One division at the start,
// none afterwards; next() past the end stays done and reads nothing.  A
// length above S_max counts as S_max.
template <int BM>
struct TileWalk {
    long long g, g_end;
    int b, j, n, tps, s_max;
    const int32_t* seq_len;
    __device__ __forceinline__ int len(int bb) const {
        const int v = seq_len[bb];
        return v < s_max ? v : s_max;
    }
    __device__ __forceinline__ void init(long long g0, long long ge, int tps_, const int32_t* sl,
                                         int s_max_) {
        g = g0;
        g_end = ge;
        tps = tps_;
        s_max = s_max_;
        seq_len = sl;
        b = static_cast<int>(g0 / tps_);
        j = static_cast<int>(g0 - static_cast<long long>(b) * tps_);
        n = g < g_end ? len(b) : 0;
        settle();
    }
    __device__ __forceinline__ void settle() {
        while (g < g_end && j * BM >= n) {
            g += tps - j;
            ++b;
            j = 0;
            if (g < g_end) n = len(b);
        }
    }
    __device__ __forceinline__ bool done() const { return g >= g_end; }
    __device__ __forceinline__ void next() {
        ++g;
        if (++j == tps) {
            j = 0;
            ++b;
            if (g < g_end) n = len(b);
        }
        settle();
    }
};

template <int H_I>
__global__ void __launch_bounds__(512, 1)
    k_index_score_decode(const __grid_constant__ CUtensorMap tm_k,
                         const __nv_bfloat16* __restrict__ qg, const __nv_bfloat16* __restrict__ w,
                         const float* __restrict__ kscale, const int32_t* __restrict__ seq_len,
                         int B, int S_max, int tps, float* __restrict__ scores, long long ld,
                         uint32_t* __restrict__ hist, int* __restrict__ err) {
    using S = DecodeShape<H_I>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sA = smem + S::OFF_A;
    uint8_t* sB = smem + S::OFF_B;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint64_t* a_full = bars;                    // [A_ST] key tile landed (TMA tx)
    uint64_t* a_empty = a_full + S::A_ST;       // [A_ST] key tile consumed (MMA commit)
    uint64_t* acc_full = a_empty + S::A_ST;     // [NACC]
    uint64_t* acc_empty = acc_full + S::NACC;   // [NACC]
    uint64_t* q_full = acc_empty + S::NACC;     // [2] hi / lo written (query warps)
    uint64_t* q_empty = q_full + 2;             // [2] hi / lo no longer read (MMA commit)
    uint64_t* q_max = q_empty + 2;              // query warps' max|q| reduction
    uint64_t* done_bar = q_max + 1;
    uint32_t* qred = reinterpret_cast<uint32_t*>(smem + S::OFF_QRED);  // [2][4]
    uint8_t* seq_ring = smem + S::OFF_W;
    uint32_t* sh_hist = reinterpret_cast<uint32_t*>(smem + S::OFF_HIST);  // [2][kKeyBins]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long total = static_cast<long long>(B) * tps;
    const long long g_begin = total * blockIdx.x / gridDim.x;
    const long long g_end = total * (blockIdx.x + 1) / gridDim.x;
    // as a programmatic dependent: nothing is read before the previous kernel completes
    griddep_wait();
    griddep_launch_dependents();

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        if (smem_u32(smem) & 1023u) {
            *abort_flag = 1;
            atomicCAS(err, 0, kDevSmemMisaligned);
        }
        for (int i = 0; i < S::A_ST; ++i) {
            mbar_init(&a_full[i], 1);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < S::NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 8);  // every epilogue warp
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 4);  // one arrival per query warp
            mbar_init(&q_empty[i], 1);
        }
        mbar_init(q_max, 4);
        mbar_init(done_bar, 1);
        for (int i = 0; i < S::SEQ_RING; ++i)
            *reinterpret_cast<volatile int*>(seq_ring + i * S::SEQ_BYTES) = -1;
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
    }
    if (hist != nullptr)
        for (int i = threadIdx.x; i < 2 * kKeyBins; i += blockDim.x) sh_hist[i] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool start_ok = (*abort_flag == 0);

    if (warp == 0 && lane == 0 && start_ok) {
        // ------------------------------------------------ TMA producer
        int st = 0;
        uint32_t ph = 0;
        uint32_t used = 0, last_ph = 0;  // per stage: loaded at all, parity of the last load
        TileWalk<S::BM> tw;
        for (tw.init(g_begin, g_end, tps, seq_len, S_max); !tw.done(); tw.next()) {
            if (!mbar_wait(&a_empty[st], ph ^ 1, abort_flag, err, kDevTimeoutProducer)) break;
            // rows past the end of the cache are zero-filled by TMA, rows past
            // seq_len[b] are read but never stored
            const int row0 = tw.b * S_max + tw.j * S::BM;
            mbar_arrive_expect_tx(&a_full[st], S::A_BYTES);
            tma_load_2d(sA + st * S::A_BYTES, &tm_k, &a_full[st], 0, row0);
            used |= 1u << st;
            last_ph = (last_ph & ~(1u << st)) | (ph << st);
            if (++st == S::A_ST) {
                st = 0;
                ph ^= 1;
            }
        }
        for (int i = 0; i < S::A_ST; ++i)
            if ((used >> i) & 1) mbar_wait_drain(&a_full[i], (last_ph >> i) & 1);
    } else if (warp == 1 && lane == 0 && start_ok) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t IDESC = idesc_e4m3_f32(128, S::ACC_COLS);
        int st = 0, acc = 0, qb = 0;
        uint32_t ph = 0, q_it = 0;
        uint32_t acc_ph = 0;  // bit a: parity of accumulator a's next use
        int cur_b = -1;
        TileWalk<S::BM> tw;
        for (tw.init(g_begin, g_end, tps, seq_len, S_max); !tw.done(); tw.next()) {
            if (tw.b != cur_b) {
                if (cur_b >= 0) umma_commit(&q_empty[qb]);  // previous hi / lo no longer read
                qb = static_cast<int>(q_it & 1);
                if (!mbar_wait(&q_full[qb], (q_it >> 1) & 1, abort_flag, err, kDevTimeoutMma)) break;
                ++q_it;
                cur_b = tw.b;
            }
            if (!mbar_wait(&a_full[st], ph, abort_flag, err, kDevTimeoutMma)) break;
            if (!mbar_wait(&acc_empty[acc], ((acc_ph >> acc) & 1) ^ 1, abort_flag, err,
                           kDevTimeoutMma))
                break;
            tc_fence_after();
            const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * 2 * S::ACC_COLS);
            const uint32_t a0 = smem_u32(sA + st * S::A_BYTES);
            const uint32_t b0 = smem_u32(sB + qb * S::B_BUF);  // hi rows, then lo rows
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f8(d_tmem + hf * S::ACC_COLS, sdesc_k_sw128(a0 + hf * S::A_HALF + kk * 32),
                            sdesc_k_sw128(b0 + kk * 32), IDESC, kk != 0 ? 1u : 0u);
            umma_commit(&acc_full[acc]);
            umma_commit(&a_empty[st]);
            acc_ph ^= 1u << acc;
            if (++acc == S::NACC) acc = 0;
            if (++st == S::A_ST) {
                st = 0;
                ph ^= 1;
            }
        }
        umma_commit(done_bar);
        if (!mbar_wait_drain(done_bar, 0)) atomicCAS(err, 0, kDevTimeoutDrain);
    } else if (warp >= 4 && warp < 8 && start_ok) {
        // ------------------------------------------------ query hi / lo
        const int t = threadIdx.x - 128;  // 0..127
        const int qw = t >> 5;
        constexpr int NCH = H_I * 8 / 128;  // 16-element chunks per thread
        uint32_t q_it = 0;
        int cur_b = -1;
        TileWalk<S::BM> tw;
        for (tw.init(g_begin, g_end, tps, seq_len, S_max); !tw.done(); tw.next()) {
            if (tw.b == cur_b) continue;
            cur_b = tw.b;
            const int qb = static_cast<int>(q_it & 1);
            const uint32_t par = q_it & 1;
            bool ok = mbar_wait(&q_empty[qb], ((q_it >> 1) & 1) ^ 1, abort_flag, err,
                                kDevTimeoutEpilogue);
            if (!__all_sync(0xffffffffu, ok)) break;
            // chunk c = t + 128 i: head h = c >> 3, elements 16 (c & 7) .. +15
            const uint4* qv = reinterpret_cast<const uint4*>(qg + static_cast<size_t>(cur_b) * H_I * 128);
            uint4 v[NCH][2];
            uint32_t mx = 0;
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const int c = t + 128 * i;
                v[i][0] = __ldg(qv + 2 * c);
                v[i][1] = __ldg(qv + 2 * c + 1);
            }
            // warp 0 also fetches w[b,:] now, so its latency overlaps q's
            float wv[(H_I + 31) / 32];
            if (qw == 0)
#pragma unroll
                for (int r = 0; r < (H_I + 31) / 32; ++r)
                    wv[r] = __bfloat162float(w[static_cast<size_t>(cur_b) * H_I + r * 32 + lane]);
#pragma unroll
            for (int i = 0; i < NCH; ++i)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t w4[4] = {v[i][u].x, v[i][u].y, v[i][u].z, v[i][u].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        mx = max(mx, max(w4[e] & 0x7FFFu, (w4[e] >> 16) & 0x7FFFu));
                }
            mx = __reduce_max_sync(0xffffffffu, mx);
            if (lane == 0) {
                qred[par * 4 + qw] = mx;
                mbar_arrive(q_max);
            }
            ok = mbar_wait(q_max, par, abort_flag, err, kDevTimeoutEpilogue);
            if (!__all_sync(0xffffffffu, ok)) break;
            uint32_t M = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) M = max(M, qred[par * 4 + i]);
            const int sh = q_shift_of_max(M);
            const float up = __int_as_float((127 + sh) << 23);
            uint8_t* hi_base = sB + qb * S::B_BUF;
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const int c = t + 128 * i, h = c >> 3, c16 = c & 7;
                const uint32_t* w8 = reinterpret_cast<const uint32_t*>(&v[i][0]);
                uint32_t hi4[4], lo4[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {  // 4 elements per output word
                    uint32_t hw = 0, lw = 0;
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const uint32_t bb = w8[2 * p + e2];
                        const float x0 = __uint_as_float(bb << 16) * up;
                        const float x1 = __uint_as_float(bb & 0xFFFF0000u) * up;
                        const uint32_t hp = e4m3x2_of(x0, x1);
                        const float2 hf = float2_of_e4m3x2(hp);
                        const uint32_t lp = e4m3x2_of(x0 - hf.x, x1 - hf.y);
                        hw |= hp << (16 * e2);
                        lw |= lp << (16 * e2);
                    }
                    hi4[p] = hw;
                    lo4[p] = lw;
                }
                const int off = h * 128 + ((c16 ^ (h & 7)) << 4);
                *reinterpret_cast<uint4*>(hi_base + off) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                *reinterpret_cast<uint4*>(hi_base + S::B_HALF + off) =
                    make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
            }
            // generic-proxy writes must be visible to the tensor core
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_full[qb]);
            if (qw == 0) {
                // publish w[b,:] and 2^-s for the epilogue: payload first, tag b
                // last (the epilogue reaches this sequence only after the MMA
                // consumed its q)
                uint8_t* ent = seq_ring + (q_it % S::SEQ_RING) * S::SEQ_BYTES;
                float* wr = reinterpret_cast<float*>(ent + 16);
#pragma unroll
                for (int r = 0; r < (H_I + 31) / 32; ++r) wr[r * 32 + lane] = wv[r];
                if (lane == 0) reinterpret_cast<float*>(ent)[1] = __int_as_float((127 - sh) << 23);
                __threadfence_block();
                __syncwarp();
                if (lane == 0) *reinterpret_cast<volatile int*>(ent) = cur_b;
            }
            ++q_it;
        }
    } else if (warp >= 8 && start_ok) {
        // ------------------------------------------------ epilogue
        const int hf = (warp - 8) >> 2;  // which 128-key half of every tile
        const int lq = warp & 3;         // TMEM lanes 32 lq .. 32 lq + 31
        const int key = hf * 128 + lq * 32 + lane;  // this thread's key within a tile
        const float* wW = nullptr;  // w[b,:] of the current sequence, in the ring
        uint32_t e_it = 0;          // sequences entered so far
        int acc = 0;
        uint32_t acc_ph = 0;  // bit a: parity of accumulator a's next use
        int cur_b = -1;
        float q_unscale = 1.f;  // 2^-s of the current sequence's q
        // this thread's per-token scales are prefetched SC_RING-1 tiles ahead
        // (walker `tp`) with cp.async into a per-thread shared-memory ring
        // (zero past the sequence end)
        const uint32_t sc_ring = smem_u32(smem + S::OFF_SC) + key * 4;
        TileWalk<S::BM> tw, tp;
        tw.init(g_begin, g_end, tps, seq_len, S_max);
        tp.init(g_begin, g_end, tps, seq_len, S_max);
        // the sequences of this CTA's first and last (sequence, tile) pair:
        // their score counts gather in shared memory (the others are this
        // CTA's alone and go straight to hist)
        const int b_first = static_cast<int>(g_begin / tps);
        const int b_last = g_end > g_begin ? static_cast<int>((g_end - 1) / tps) : b_first;
        auto prefetch_scale = [&](int slot) {
            if (!tp.done()) {
                const int s = tp.j * S::BM + key;
                const bool ok = s < tp.n;
                const float* src = kscale + static_cast<long long>(tp.b) * S_max + (ok ? s : 0);
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(
                                 sc_ring + slot * S::BM * 4),
                             "l"(src), "r"(ok ? 4 : 0)
                             : "memory");
                tp.next();
            }
            cp_async_commit();
        };
        int it = 0;
        for (int p = 0; p < S::SC_RING - 1; ++p) prefetch_scale(p);
        for (; !tw.done(); tw.next()) {
            prefetch_scale((it + S::SC_RING - 1) % S::SC_RING);
            const int b = tw.b, n = tw.n;
            const int s = tw.j * S::BM + key;
            if (b != cur_b) {
                // the query warps published this sequence's entry before its q
                // reached the tensor core; the tag makes the read self-checking
                const uint8_t* ent = seq_ring + (e_it % S::SEQ_RING) * S::SEQ_BYTES;
                bool seen = *reinterpret_cast<const volatile int*>(ent) == b;
                if (!seen) {  // bounded: gives up on the CTA's abort flag or after the limit
                    const long long t0 = clock64();
                    while (!(seen = *reinterpret_cast<const volatile int*>(ent) == b)) {
                        if (*abort_flag) break;
                        if (clock64() - t0 > kWaitLimitCycles) {
                            *abort_flag = 1;
                            atomicCAS(err, 0, kDevTimeoutEpilogue);
                            break;
                        }
                        __nanosleep(64);
                    }
                }
                if (!__all_sync(0xffffffffu, seen)) break;
                __threadfence_block();
                q_unscale = reinterpret_cast<const volatile float*>(ent)[1];
                wW = reinterpret_cast<const float*>(ent + 16);
                ++e_it;
                cur_b = b;
            }
            bool got = mbar_wait(&acc_full[acc], (acc_ph >> acc) & 1, abort_flag, err,
                                 kDevTimeoutEpilogue);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16) +
                                   static_cast<uint32_t>((2 * acc + hf) * S::ACC_COLS);
            uint64_t p2[2] = {0, 0};  // two packed partial sums (heads h = 0, 1 mod 4; 2, 3 mod 4)
#pragma unroll
            for (int h0 = 0; h0 < H_I; h0 += 32) {  // 32 heads: their hi and lo columns
                uint32_t vh[32], vl[32];
                tmem_ld32(taddr + h0, vh);
                tmem_ld32(taddr + H_I + h0, vl);
                tmem_ld_wait();
                if (h0 + 32 == H_I) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[acc]);
                }
#pragma unroll
                for (int h = 0; h < 32; h += 4) {
                    const ulonglong2 w2 = *reinterpret_cast<const ulonglong2*>(wW + h0 + h);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float2 x = f2_unpack(
                            f2_add(f2_pack(__uint_as_float(vh[h + 2 * u]), __uint_as_float(vh[h + 2 * u + 1])),
                                   f2_pack(__uint_as_float(vl[h + 2 * u]), __uint_as_float(vl[h + 2 * u + 1]))));
                        p2[u] = f2_fma(u ? w2.y : w2.x, f2_pack(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)), p2[u]);
                    }
                }
            }
            const float2 pa = f2_unpack(p2[0]), pb = f2_unpack(p2[1]);
            const float p[4] = {pa.x, pa.y, pb.x, pb.y};
            cp_async_wait<S::SC_RING - 1>();  // this tile's scale has landed
            float sc;
            asm volatile("ld.shared.f32 %0, [%1];"
                         : "=f"(sc)
                         : "r"(sc_ring + (it % S::SC_RING) * S::BM * 4));
            const float val = (sc * q_unscale) * ((p[0] + p[1]) + (p[2] + p[3]));
            if (s < n) scores[static_cast<long long>(b) * ld + s] = val;
            if (hist != nullptr && s < n) {
                // b is the same for the whole tile: the slot is chosen once
                const uint32_t bin = order_key(val) >> kKeyBinShift;
                if (b == b_first || b == b_last)
                    atomicAdd(&sh_hist[(b == b_first ? 0 : kKeyBins) + bin], 1u);
                else
                    atomicAdd(&hist[static_cast<long long>(b) * kKeyBins + bin], 1u);
            }
            acc_ph ^= 1u << acc;
            if (++acc == S::NACC) acc = 0;
            ++it;
        }
        cp_async_wait<0>();  // no prefetch may still be landing at exit
        if (hist != nullptr) {
            // every epilogue warp leaves the tile loop (also on an abort) and
            // meets here; then the shared counts go out, one add per bin
            asm volatile("bar.sync 1, %0;" ::"n"(256) : "memory");
            const int et = threadIdx.x - 256;  // 0..255
            for (int i = et; i < 2 * kKeyBins; i += 256) {
                const uint32_t c = sh_hist[i];
                const int bb = i < kKeyBins ? b_first : b_last;
                if (c != 0 && !(i >= kKeyBins && b_last == b_first))
                    atomicAdd(&hist[static_cast<long long>(bb) * kKeyBins + (i % kKeyBins)], c);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_COLS);
    }
}

template <int H_I>
static int launch_decode_t(ic_ctx* ctx, const void* q, const void* w, const uint8_t* kI8,
                           const float* kI_scale, const int32_t* seq_len, int B, int S_max,
                           float* scores, int64_t ld, uint32_t* hist, cudaStream_t stream) {
    using S = DecodeShape<H_I>;
    static PerDeviceOnce attr_once;
    cudaError_t ea = attr_once.run(ctx->device, [] {
        return cudaFuncSetAttribute(k_index_score_decode<H_I>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
    });
    if (ea != cudaSuccess) return cuda_fail(ctx, ea, "cudaFuncSetAttribute(index_decode)");
    // tile row coordinates are 32-bit
    if (static_cast<long long>(B) * S_max + S::BM > 0x7FFFFFFFll)
        return fail(ctx, IC_ERR_SHAPE, "decode index: B*S_max=%lld too large",
                    static_cast<long long>(B) * S_max);
    CUtensorMap tm_k;
    int rc = make_tmap_u8_2d(ctx, &tm_k, kI8, static_cast<uint64_t>(B) * S_max, 128, 128, S::BM,
                             true);
    if (rc) return rc;
    const int tps = (S_max + S::BM - 1) / S::BM;
    const long long total = static_cast<long long>(B) * tps;
    const int grid = total < ctx->num_sms ? static_cast<int>(total) : ctx->num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(512, 1, 1);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    unsigned int na = 0;
    add_pdl_attr(ctx, attr, na);
    cfg.attrs = attr;
    cfg.numAttrs = na;
    LaunchScope ls(ctx, IC_K_INDEX_SCORE_DECODE, stream);
    cudaLaunchKernelEx(&cfg, k_index_score_decode<H_I>, tm_k, static_cast<const __nv_bfloat16*>(q),
                       static_cast<const __nv_bfloat16*>(w), kI_scale, seq_len, B, S_max, tps,
                       scores, static_cast<long long>(ld), hist, ctx->dev_err);
    cudaError_t e = ls.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "index_score_decode launch");
    return IC_OK;
}

int launch_index_score_decode(ic_ctx* ctx, const void* q, const void* w, const uint8_t* kI8,
                              const float* kI_scale, const int32_t* seq_len, int B, int S_max,
                              int H_I, int d_I, float* scores, int64_t ld, cudaStream_t stream,
                              uint32_t* hist) {
    if (d_I != 128) return fail(ctx, IC_ERR_UNSUPPORTED, "decode index: d_I=%d (need 128)", d_I);
    if (H_I == 64)
        return launch_decode_t<64>(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, scores, ld, hist,
                                   stream);
    if (H_I == 32)
        return launch_decode_t<32>(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, scores, ld, hist,
                                   stream);
    return fail(ctx, IC_ERR_UNSUPPORTED, "decode index: H_I=%d (need 32 or 64)", H_I);
}

}  // namespace ic
