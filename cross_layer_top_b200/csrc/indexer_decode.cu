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
// Design (sm_100a), one persistent CTA per SM, HBM-bound by construction:
//  * warp 0 (TMA): streams raw e4m3 key tiles (128 keys x 128 B, one
//    contiguous 16 KB block each, so one bulk copy) through a 5-deep ring,
//    and the sequence's q rows (bf16, 128-byte swizzle, a tensor copy)
//    when the sequence changes;
//  * warps 4..11 (convert): widen each e4m3 tile to bf16 — exact, every e4m3
//    value is a bf16 value — and write it in the K-major 128-byte-swizzle
//    layout the tensor core reads, then fence the async proxy;
//  * warp 1 (MMA): UMMA M=128 keys x N=H_I heads x K=128, fp32 in TMEM, four
//    accumulators in flight;
//  * warps 12..15 (epilogue): the thread owning TMEM lane s applies ReLU,
//    the w weights, the head sum and the per-token scale, and stores I[b,s].
// Each CTA scans a contiguous range of (sequence, key tile) pairs, so q is
// reloaded only when its range crosses into the next sequence.  All waits
// are bounded.
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

template <int H_I>
struct DecodeShape {
    static constexpr int BM = 128;          // keys per tile
    static constexpr int DI = 128;          // d_I
    static constexpr int RAW = BM * DI;     // e4m3 tile bytes
    static constexpr int RAW_ST = 5;
    static constexpr int A_ATOM = BM * 128; // bf16 64-column slice
    static constexpr int A_STAGE = 2 * A_ATOM;
    static constexpr int A_ST = 3;
    static constexpr int B_ATOM = H_I * 128;
    static constexpr int B_BYTES = 2 * B_ATOM;
    static constexpr int NACC = 4;
    static constexpr int TMEM_COLS = NACC * H_I < 32 ? 32 : NACC * H_I;
    static constexpr int W_BYTES = 4 * H_I * 4;  // per epilogue warp
    static constexpr int SC_RING = 4;             // scale prefetch depth (tiles)
    static constexpr int SC_BYTES = SC_RING * BM * 4;
    static constexpr int BAR_BYTES = 256;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + A_ST * A_STAGE;
    static constexpr int OFF_RAW = OFF_B + B_BYTES;
    static constexpr int OFF_W = OFF_RAW + RAW_ST * RAW;
    static constexpr int OFF_SC = OFF_W + W_BYTES;
    static constexpr int OFF_BAR = OFF_SC + SC_BYTES;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES;
    static_assert(SMEM <= 232448, "shared memory budget");
};

// Two e4m3 bytes (low bytes of the two 16-bit lanes of y) -> bf16x2, exactly.
// The e4m3 sign goes to bit 15 and its 7 exponent/mantissa bits to bits
// 10..4, i.e. a bf16 whose exponent field is the e4m3 exponent field
// unbiased: value * 2^-120 (for an e4m3 subnormal, the matching bf16
// subnormal).  One bf16x2 multiply by 2^120 restores the value; it is exact
// (a power-of-two scaling into the normal range).  The e4m3 NaN bytes
// (0x7F, 0xFF) are not NaN afterwards (+-480); caches hold none.
__device__ __forceinline__ uint32_t e4m3x2_lanes_to_bf16x2(uint32_t y) {
    // (low 7 bits << 4) | (sign << 8) == (y << 4) + sign * (256 - 16)
    const uint32_t bits = (y & 0x00800080u) * 240u + (y << 4);
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&bits);
    const __nv_bfloat162 s = __halves2bfloat162(__ushort_as_bfloat16(0x7B80),
                                                __ushort_as_bfloat16(0x7B80));  // 2^120
    const __nv_bfloat162 r = __hmul2(v, s);
    return *reinterpret_cast<const uint32_t*>(&r);
}

// 16 e4m3 values (one 16-byte chunk) -> 16 bf16 values, exactly.
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4 in, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = e4m3x2_lanes_to_bf16x2(__byte_perm(w[i], 0u, 0x4140));      // bytes 0, 1
        o[2 * i + 1] = e4m3x2_lanes_to_bf16x2(__byte_perm(w[i], 0u, 0x4342));  // bytes 2, 3
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Walks a CTA's contiguous range of (sequence b, key tile j) pairs in order,
// visiting only tiles that hold candidates (j * BM < seq_len[b]) and
// skipping a sequence's empty tail in one step.  One division at the start,
// none afterwards.
template <int BM>
struct TileWalk {
    long long g, g_end;
    int b, j, n, tps;
    const int32_t* seq_len;
    __device__ __forceinline__ void init(long long g0, long long ge, int tps_, const int32_t* sl) {
        g = g0;
        g_end = ge;
        tps = tps_;
        seq_len = sl;
        b = static_cast<int>(g0 / tps_);
        j = static_cast<int>(g0 - static_cast<long long>(b) * tps_);
        n = g < g_end ? seq_len[b] : 0;
        settle();
    }
    __device__ __forceinline__ void settle() {
        while (g < g_end && j * BM >= n) {
            g += tps - j;
            ++b;
            j = 0;
            if (g < g_end) n = seq_len[b];
        }
    }
    __device__ __forceinline__ bool done() const { return g >= g_end; }
    __device__ __forceinline__ void next() {
        ++g;
        if (++j == tps) {
            j = 0;
            ++b;
            if (g < g_end) n = seq_len[b];
        }
        settle();
    }
};

template <int H_I>
__global__ void __launch_bounds__(512, 1)
    k_index_score_decode(const __grid_constant__ CUtensorMap tm_q,
                         const uint8_t* __restrict__ k8,
                         const __nv_bfloat16* __restrict__ w, const float* __restrict__ kscale,
                         const int32_t* __restrict__ seq_len, int B, int S_max, int tps,
                         float* __restrict__ scores, long long ld, int* __restrict__ err) {
    using S = DecodeShape<H_I>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sA = smem + S::OFF_A;
    uint8_t* sB = smem + S::OFF_B;
    uint8_t* sRaw = smem + S::OFF_RAW;
    float* sW = reinterpret_cast<float*>(smem + S::OFF_W);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint64_t* raw_full = bars;                  // [RAW_ST]
    uint64_t* raw_empty = raw_full + S::RAW_ST; // [RAW_ST]
    uint64_t* a_full = raw_empty + S::RAW_ST;   // [A_ST]
    uint64_t* a_empty = a_full + S::A_ST;       // [A_ST]
    uint64_t* acc_full = a_empty + S::A_ST;     // [NACC]
    uint64_t* acc_empty = acc_full + S::NACC;   // [NACC]
    uint64_t* q_full = acc_empty + S::NACC;
    uint64_t* q_empty = q_full + 1;
    uint64_t* done_bar = q_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long total = static_cast<long long>(B) * tps;
    const long long g_begin = total * blockIdx.x / gridDim.x;
    const long long g_end = total * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        if (smem_u32(smem) & 1023u) {
            *abort_flag = 1;
            atomicCAS(err, 0, kDevSmemMisaligned);
        }
        for (int i = 0; i < S::RAW_ST; ++i) {
            mbar_init(&raw_full[i], 1);
            mbar_init(&raw_empty[i], 8);  // one arrival per converter warp
        }
        for (int i = 0; i < S::A_ST; ++i) {
            mbar_init(&a_full[i], 8);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < S::NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(done_bar, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool start_ok = (*abort_flag == 0);

    if (warp == 0 && lane == 0 && start_ok) {
        // ------------------------------------------------ TMA producer
        int rs = 0;
        uint32_t rph = 0, q_it = 0;
        int last_ph[S::RAW_ST];
#pragma unroll
        for (int i = 0; i < S::RAW_ST; ++i) last_ph[i] = -1;
        int q_last = -1, cur_b = -1;
        TileWalk<S::BM> tw;
        for (tw.init(g_begin, g_end, tps, seq_len); !tw.done(); tw.next()) {
            const int b = tw.b, j = tw.j;
            if (b != cur_b) {
                if (!mbar_wait(q_empty, (q_it & 1) ^ 1, abort_flag, err, kDevTimeoutProducer)) break;
                mbar_arrive_expect_tx(q_full, S::B_BYTES);
                tma_load_2d(sB, &tm_q, q_full, 0, b * H_I);
                tma_load_2d(sB + S::B_ATOM, &tm_q, q_full, 64, b * H_I);
                q_last = q_it & 1;
                ++q_it;
                cur_b = b;
            }
            if (!mbar_wait(&raw_empty[rs], rph ^ 1, abort_flag, err, kDevTimeoutProducer)) break;
            // the tile's 128 key rows are one contiguous block: a single bulk
            // copy, clamped at the end of the cache (rows past it stay stale
            // and are never stored)
            const long long row0 = static_cast<long long>(b) * S_max + j * S::BM;
            const long long left = static_cast<long long>(B) * S_max - row0;
            const uint32_t bytes = static_cast<uint32_t>(left < S::BM ? left : S::BM) * S::DI;
            mbar_arrive_expect_tx(&raw_full[rs], bytes);
            bulk_load(smem_u32(sRaw + rs * S::RAW), k8 + row0 * S::DI, bytes, &raw_full[rs]);
            last_ph[rs] = static_cast<int>(rph);
            if (++rs == S::RAW_ST) {
                rs = 0;
                rph ^= 1;
            }
        }
        for (int i = 0; i < S::RAW_ST; ++i)
            if (last_ph[i] >= 0) mbar_wait_drain(&raw_full[i], static_cast<uint32_t>(last_ph[i]));
        if (q_last >= 0) mbar_wait_drain(q_full, static_cast<uint32_t>(q_last));
    } else if (warp == 1 && lane == 0 && start_ok) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t IDESC = idesc_bf16_f32(S::BM, H_I);
        int as = 0, acc = 0;
        uint32_t aph = 0, q_it = 0;
        uint32_t acc_it[S::NACC] = {0, 0, 0, 0};
        int cur_b = -1;
        bool ok = true;
        TileWalk<S::BM> tw;
        for (tw.init(g_begin, g_end, tps, seq_len); !tw.done() && ok; tw.next()) {
            const int b = tw.b;
            if (b != cur_b) {
                if (cur_b >= 0) umma_commit(q_empty);  // previous q no longer read
                if (!mbar_wait(q_full, q_it & 1, abort_flag, err, kDevTimeoutMma)) break;
                ++q_it;
                cur_b = b;
            }
            if (!mbar_wait(&a_full[as], aph, abort_flag, err, kDevTimeoutMma)) break;
            if (!mbar_wait(&acc_empty[acc], (acc_it[acc] & 1) ^ 1, abort_flag, err,
                           kDevTimeoutMma)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * H_I);
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad =
                        sdesc_k_sw128(smem_u32(sA + as * S::A_STAGE + k * S::A_ATOM + kk * 32));
                    const uint64_t bd = sdesc_k_sw128(smem_u32(sB + k * S::B_ATOM + kk * 32));
                    umma_bf16(d_tmem, ad, bd, IDESC, (k | kk) != 0 ? 1u : 0u);
                }
            umma_commit(&acc_full[acc]);
            umma_commit(&a_empty[as]);
            ++acc_it[acc];
            if (++acc == S::NACC) acc = 0;
            if (++as == S::A_ST) {
                as = 0;
                aph ^= 1;
            }
        }
        umma_commit(done_bar);
        if (!mbar_wait_drain(done_bar, 0)) atomicCAS(err, 0, kDevTimeoutDrain);
    } else if (warp >= 4 && warp < 12 && start_ok) {
        // ------------------------------------------------ e4m3 -> bf16
        const int t = threadIdx.x - 128;  // 0..255
        int rs = 0, as = 0;
        uint32_t rph = 0, aph = 0;
        bool ok = true;
        TileWalk<S::BM> tw;
        for (tw.init(g_begin, g_end, tps, seq_len); !tw.done() && ok; tw.next()) {
            bool got = mbar_wait(&raw_full[rs], rph, abort_flag, err, kDevTimeoutEpilogue);
            got = got && mbar_wait(&a_empty[as], aph ^ 1, abort_flag, err, kDevTimeoutEpilogue);
            got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
            const uint8_t* raw = sRaw + rs * S::RAW;
            uint8_t* dst = sA + as * S::A_STAGE;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = i * 256 + t;       // 16-byte chunk id in the raw tile
                const int row = c >> 3, c8 = c & 7;
                const uint4 v = *reinterpret_cast<const uint4*>(raw + c * 16);
                uint4 lo, hi;
                e4m3x16_to_bf16(v, lo, hi);
                uint8_t* atom = dst + (c8 >> 2) * S::A_ATOM + row * 128;
                const int ch = 2 * (c8 & 3);
                *reinterpret_cast<uint4*>(atom + ((ch ^ (row & 7)) << 4)) = lo;
                *reinterpret_cast<uint4*>(atom + (((ch + 1) ^ (row & 7)) << 4)) = hi;
            }
            // generic-proxy writes must be visible to the tensor core; one
            // arrival per warp keeps the barriers' arrival traffic small
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if ((threadIdx.x & 31) == 0) {
                mbar_arrive(&a_full[as]);
                mbar_arrive(&raw_empty[rs]);
            }
            if (++rs == S::RAW_ST) {
                rs = 0;
                rph ^= 1;
            }
            if (++as == S::A_ST) {
                as = 0;
                aph ^= 1;
            }
        }
    } else if (warp >= 12 && start_ok) {
        // ------------------------------------------------ epilogue
        const int lq = warp & 3;
        float* wW = sW + lq * H_I;
        int acc = 0;
        uint32_t acc_it[S::NACC] = {0, 0, 0, 0};
        int cur_b = -1;
        // this thread's per-token scales are prefetched SC_RING-1 tiles ahead
        // (walker `tp`) with cp.async into a per-thread shared-memory ring
        // (zero past the sequence end), so no register waits on a global load
        const uint32_t sc_ring = smem_u32(smem + S::OFF_SC) + (lq * 32 + lane) * 4;
        TileWalk<S::BM> tw, tp;
        tw.init(g_begin, g_end, tps, seq_len);
        tp.init(g_begin, g_end, tps, seq_len);
        auto prefetch_scale = [&](int slot) {
            if (!tp.done()) {
                const int s = tp.j * S::BM + lq * 32 + lane;
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
            const int b = tw.b, j = tw.j, n = tw.n;
            if (b != cur_b) {
                __syncwarp();
                for (int h = lane; h < H_I; h += 32)
                    wW[h] = __bfloat162float(w[static_cast<size_t>(b) * H_I + h]);
                __syncwarp();
                cur_b = b;
            }
            const int s = j * S::BM + lq * 32 + lane;
            bool got = mbar_wait(&acc_full[acc], acc_it[acc] & 1, abort_flag, err,
                                 kDevTimeoutEpilogue);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            tc_fence_after();
            const uint32_t taddr =
                tmem + (static_cast<uint32_t>(lq * 32) << 16) + static_cast<uint32_t>(acc * H_I);
            uint32_t va[32], vb[32];
            tmem_ld32(taddr, va);
            if (H_I == 64) tmem_ld32(taddr + 32, vb);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int h = 0; h < H_I; h += 4) {
                const float4 wv = *reinterpret_cast<const float4*>(wW + h);
                const uint32_t* src = h < 32 ? va : vb;
                p[0] = fmaf(wv.x, fmaxf(__uint_as_float(src[(h + 0) & 31]), 0.f), p[0]);
                p[1] = fmaf(wv.y, fmaxf(__uint_as_float(src[(h + 1) & 31]), 0.f), p[1]);
                p[2] = fmaf(wv.z, fmaxf(__uint_as_float(src[(h + 2) & 31]), 0.f), p[2]);
                p[3] = fmaf(wv.w, fmaxf(__uint_as_float(src[(h + 3) & 31]), 0.f), p[3]);
            }
            cp_async_wait<S::SC_RING - 1>();  // this tile's scale has landed
            float sc;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc) : "r"(sc_ring + (it % S::SC_RING) * S::BM * 4));
            if (s < n) scores[static_cast<long long>(b) * ld + s] = sc * ((p[0] + p[1]) + (p[2] + p[3]));
            ++acc_it[acc];
            if (++acc == S::NACC) acc = 0;
            ++it;
        }
        cp_async_wait<0>();  // no prefetch may still be landing at exit
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
                           float* scores, int64_t ld, cudaStream_t stream) {
    using S = DecodeShape<H_I>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_index_score_decode<H_I>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaFuncSetAttribute(index_decode)");
        attr_set = true;
    }
    CUtensorMap tm_q;
    int rc = make_tmap_bf16_2d(ctx, &tm_q, q, static_cast<uint64_t>(B) * H_I, 128, H_I);
    if (rc) return rc;
    const int tps = (S_max + S::BM - 1) / S::BM;
    const long long total = static_cast<long long>(B) * tps;
    const int grid = total < ctx->num_sms ? static_cast<int>(total) : ctx->num_sms;
    LaunchScope ls(ctx, IC_K_INDEX_SCORE_DECODE, stream);
    k_index_score_decode<H_I><<<grid, 512, S::SMEM, stream>>>(
        tm_q, kI8, static_cast<const __nv_bfloat16*>(w), kI_scale, seq_len, B, S_max, tps,
        scores, static_cast<long long>(ld), ctx->dev_err);
    cudaError_t e = ls.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "index_score_decode launch");
    return IC_OK;
}

int launch_index_score_decode(ic_ctx* ctx, const void* q, const void* w, const uint8_t* kI8,
                              const float* kI_scale, const int32_t* seq_len, int B, int S_max,
                              int H_I, int d_I, float* scores, int64_t ld, cudaStream_t stream) {
    if (d_I != 128) return fail(ctx, IC_ERR_UNSUPPORTED, "decode index: d_I=%d (need 128)", d_I);
    if (H_I == 64)
        return launch_decode_t<64>(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, scores, ld, stream);
    if (H_I == 32)
        return launch_decode_t<32>(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, scores, ld, stream);
    return fail(ctx, IC_ERR_UNSUPPORTED, "decode index: H_I=%d (need 32 or 64)", H_I);
}

}  // namespace ic
