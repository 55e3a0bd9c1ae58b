// Prefill lightning-indexer score on tcgen05 tensor cores.
//
// Computes, for query rows t in [row_begin, row_end) and keys s <= t,
//   I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j,:] . k_I[s,:])
// The q_I and w tensors may hold a window of rows only: row t of them is at
// t - q_row0 (q_row0 = 0 when they hold every row).
// ("IndexCache：跨层复用稀疏索引，以及它为什么能被训练", §2.1, the DSA
// lightning-indexer score; "IndexCache: Accelerating Sparse Attention via
// Cross-Layer Index Reuse", §2.1: the indexer scores all preceding tokens).
//
// Design (sm_100a):
//  * The contraction is arranged "keys as M": A = a tile of 128 keys of k_I
//    (K-major, 128-byte swizzle, loaded by TMA), B = the (token, head) rows
//    of q_I for a block of query tokens (K-major, same swizzle).  One UMMA
//    (M=128, N=256, K=16, bf16 in, fp32 accumulate) gives per-head dot
//    products D[s, (t,j)] in TMEM: lane = key, column = (token, head).
//  * The epilogue thread that owns TMEM lane s therefore holds all heads of
//    (t, s) in its own registers: ReLU, the w[t,j] weighting and the sum over
//    heads run without any cross-thread reduction, and only I[t,s] (fp32)
//    is stored.  The per-head [H_I, L, L] tensor never reaches HBM.
//  * A work item is TQ = 2 * 256/H_I query tokens; its q_I block stays in
//    shared memory while the causal key tiles 0..t_last/128 stream through
//    a TMA ring.  Two 256-column TMEM accumulators ping-pong so the epilogue
//    of one overlaps the MMAs of the other.
//  * Warp roles (one CTA per SM, persistent): warp 0 = TMA producer, warp 1
//    = MMA issuer, warp 2 = TMEM allocator, warps 4.. = epilogue (8 for bf16,
//    16 for e4m3; warp w reads TMEM lanes 32*(w%4).. and column group
//    (w-4)/4 of each accumulator).
//  * Work items are handed out longest-first (latest rows first), round
//    robin over the persistent CTAs.
//  * Every mbarrier wait is bounded; on timeout the CTA aborts cleanly
//    (drains its TMA loads and MMAs, frees TMEM) and latches an error code.
#include "ic_device.cuh"
#include "ic_internal.h"

namespace ic {

// F8: e4m3 q_I / k_I (d_I = 128, one 128-byte atom per row) on kind::f8f6f4
// with per-(token, head) and per-token fp32 scales; otherwise bf16.
template <int H_I, int NATOM, bool F8 = false>
struct PrefillShape {
    static constexpr int BM = 128;                 // keys per tile (UMMA M, TMEM lanes)
    static constexpr int BN = 256;                 // (token, head) columns per accumulator
    static constexpr int NACC = 2;                 // TMEM accumulators (2 x 256 = 512 columns)
    static constexpr int TOK_PER_ACC = BN / H_I;
    static constexpr int TQ = NACC * TOK_PER_ACC;  // query tokens per work item
    static constexpr int A_ATOM = BM * 128;        // one 64-element K slice of a key tile
    static constexpr int A_STAGE = NATOM * A_ATOM;
    static constexpr int B_ATOM = BN * 128;
    static constexpr int B_ACC = NATOM * B_ATOM;
    static constexpr int B_BYTES = NACC * B_ACC;
    // epilogue warps: at the fp8 MMA rate 8 warps (two per TMEM lane
    // quarter) score too slowly, so e4m3 inputs take 16
    static constexpr int EPI = F8 ? 16 : 8;
    static constexpr int THREADS = (4 + EPI) * 32;
    static constexpr int COLS = BN / (EPI / 4);    // columns per epilogue warp and accumulator
    static constexpr int W_BYTES = 8 * 1024;       // EPI warps x NACC x COLS fp32 weights
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_CAP = 232448;
    static constexpr int KST_RAW = (SMEM_CAP - B_BYTES - W_BYTES - BAR_BYTES) / A_STAGE;
    static constexpr int KSTAGES = KST_RAW > 6 ? 6 : KST_RAW;
    static constexpr int SMEM = B_BYTES + KSTAGES * A_STAGE + W_BYTES + BAR_BYTES;
    static_assert(KSTAGES >= 2, "shared memory too small for the key ring");
    static_assert(SMEM <= SMEM_CAP, "shared memory budget");
    static_assert(64 % H_I == 0, "H_I must divide 64");
    static_assert(!F8 || NATOM == 1, "e4m3 rows of d_I = 128 are one 128-byte atom");
};

// The scoring kernel (one persistent CTA per SM, warp roles as above):
// scores of query rows [row_begin, row_end) against keys s <= t, written to
// scores[(t - row_begin) * ld + s].
template <int H_I, int NATOM, bool F8>
__global__ void __launch_bounds__(PrefillShape<H_I, NATOM, F8>::THREADS, 1)
    k_index_score_prefill(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __nv_bfloat16* __restrict__ w, const float* __restrict__ q_scale,
                          const float* __restrict__ k_scale, float* __restrict__ scores,
                          long long ld, int L, int row_begin, int row_end, int n_items,
                          int q_row0, int q_rows, int* __restrict__ err) {
    using S = PrefillShape<H_I, NATOM, F8>;
    constexpr int KST = S::KSTAGES;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sB = smem;
    uint8_t* sA = smem + S::B_BYTES;
    float* sW = reinterpret_cast<float*>(sA + KST * S::A_STAGE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sW) + S::W_BYTES);
    uint64_t* a_full = bars;
    uint64_t* a_empty = bars + KST;
    uint64_t* q_full = bars + 2 * KST;
    uint64_t* q_empty = q_full + 1;
    uint64_t* acc_full = q_full + 2;   // [2]
    uint64_t* acc_empty = q_full + 4;  // [2]
    uint64_t* done_bar = q_full + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        if (smem_u32(smem) & 1023u) {
            *abort_flag = 1;
            atomicCAS(err, 0, kDevSmemMisaligned);
        }
        for (int i = 0; i < KST; ++i) {
            mbar_init(&a_full[i], 1);
            mbar_init(&a_empty[i], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], S::EPI);  // one arrival per epilogue warp
        }
        mbar_init(done_bar, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool start_ok = (*abort_flag == 0);

    if (warp == 0 && lane == 0 && start_ok) {
        // ------------------------------------------------ TMA producer
        int st = 0;
        uint32_t ph = 0, q_it = 0;
        int last_ph[KST];
#pragma unroll
        for (int i = 0; i < KST; ++i) last_ph[i] = -1;
        int q_last = -1;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const int t0 = row_begin + (n_items - 1 - it) * S::TQ;
            const int t_last = min(t0 + S::TQ, row_end) - 1;
            const int n_tiles = t_last / S::BM + 1;
            if (!mbar_wait(q_empty, (q_it & 1) ^ 1, abort_flag, err, kDevTimeoutProducer)) {
                ok = false;
                break;
            }
            mbar_arrive_expect_tx(q_full, S::B_BYTES);
#pragma unroll
            for (int a = 0; a < S::NACC; ++a)
#pragma unroll
                for (int k = 0; k < NATOM; ++k)
                    tma_load_2d(sB + a * S::B_ACC + k * S::B_ATOM, &tm_q, q_full, k * 64,
                                (t0 - q_row0 + a * S::TOK_PER_ACC) * H_I);
            q_last = q_it & 1;
            ++q_it;
            for (int kt = 0; kt < n_tiles; ++kt) {
                if (!mbar_wait(&a_empty[st], ph ^ 1, abort_flag, err, kDevTimeoutProducer)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&a_full[st], S::A_STAGE);
#pragma unroll
                for (int k = 0; k < NATOM; ++k)
                    tma_load_2d(sA + st * S::A_STAGE + k * S::A_ATOM, &tm_k, &a_full[st], k * 64,
                                kt * S::BM);
                last_ph[st] = static_cast<int>(ph);
                if (++st == KST) {
                    st = 0;
                    ph ^= 1;
                }
            }
        }
        // No TMA write may still be landing in shared memory when the CTA exits.
        for (int i = 0; i < KST; ++i)
            if (last_ph[i] >= 0) mbar_wait_drain(&a_full[i], static_cast<uint32_t>(last_ph[i]));
        if (q_last >= 0) mbar_wait_drain(q_full, static_cast<uint32_t>(q_last));
    } else if (warp == 1 && lane == 0 && start_ok) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t IDESC = F8 ? idesc_e4m3_f32(S::BM, S::BN) : idesc_bf16_f32(S::BM, S::BN);
        int st = 0;
        uint32_t ph = 0, q_it = 0;
        uint32_t acc_it[2] = {0, 0};
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const int t0 = row_begin + (n_items - 1 - it) * S::TQ;
            const int t_last = min(t0 + S::TQ, row_end) - 1;
            const int n_tiles = t_last / S::BM + 1;
            if (!mbar_wait(q_full, q_it & 1, abort_flag, err, kDevTimeoutMma)) {
                ok = false;
                break;
            }
            ++q_it;
            tc_fence_after();
            for (int kt = 0; kt < n_tiles && ok; ++kt) {
                if (!mbar_wait(&a_full[st], ph, abort_flag, err, kDevTimeoutMma)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    if (!mbar_wait(&acc_empty[a], (acc_it[a] & 1) ^ 1, abort_flag, err,
                                   kDevTimeoutMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem + static_cast<uint32_t>(a * S::BN);
#pragma unroll
                    for (int k = 0; k < NATOM; ++k)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = sdesc_k_sw128(
                                smem_u32(sA + st * S::A_STAGE + k * S::A_ATOM + kk * 32));
                            const uint64_t bd = sdesc_k_sw128(
                                smem_u32(sB + a * S::B_ACC + k * S::B_ATOM + kk * 32));
                            // K = 16 bf16 or 32 e4m3: 32 bytes of each row either way
                            if (F8)
                                umma_f8(d_tmem, ad, bd, IDESC, (k | kk) != 0 ? 1u : 0u);
                            else
                                umma_bf16(d_tmem, ad, bd, IDESC, (k | kk) != 0 ? 1u : 0u);
                        }
                    umma_commit(&acc_full[a]);
                    ++acc_it[a];
                }
                if (!ok) break;
                umma_commit(&a_empty[st]);
                if (++st == KST) {
                    st = 0;
                    ph ^= 1;
                }
            }
            if (!ok) break;
            umma_commit(q_empty);
        }
        // Every MMA this thread issued completes before TMEM is released.
        umma_commit(done_bar);
        if (!mbar_wait_drain(done_bar, 0)) atomicCAS(err, 0, kDevTimeoutDrain);
    } else if (warp >= 4 && start_ok) {
        // ------------------------------------------------ epilogue
        constexpr int COLS = S::COLS;
        constexpr int CPL = COLS / 32;        // staged weights per lane and accumulator
        constexpr int NCHUNK = COLS / 32;     // 32-column TMEM loads per accumulator
        const int ew = warp - 4;  // 0..EPI-1
        const int lq = warp & 3;  // TMEM lane quarter
        const int cg = ew >> 2;   // column group of each accumulator
        float* wW = sW + ew * 2 * COLS;  // this warp's weights: [acc][COLS columns]
        uint32_t acc_it[2] = {0, 0};
        bool ok = true;
        constexpr int TOK_PER_HALF = COLS / H_I;  // tokens in this warp's columns
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const int t0 = row_begin + (n_items - 1 - it) * S::TQ;
            const int t_last = min(t0 + S::TQ, row_end) - 1;
            const int n_tiles = t_last / S::BM + 1;
            // weights of this warp's columns, widened to fp32 (private copy);
            // e4m3 inputs fold the query's (token, head) scale in: it is > 0,
            // so it commutes with ReLU
            __syncwarp();
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const int tok0 = t0 + a * S::TOK_PER_ACC + cg * TOK_PER_HALF;
#pragma unroll
                for (int q = 0; q < CPL; ++q) {
                    const int c = lane * CPL + q;  // column within the group
                    const int tq = tok0 + c / H_I - q_row0;  // row in the q_I / w window
                    const size_t wi = static_cast<size_t>(tq) * H_I + (c % H_I);
                    float wv = tq < q_rows ? __bfloat162float(w[wi]) : 0.f;
                    if (F8 && tq < q_rows) wv *= q_scale[wi];
                    wW[a * COLS + c] = wv;
                }
            }
            __syncwarp();
            for (int kt = 0; kt < n_tiles && ok; ++kt) {
                const int s = kt * S::BM + lq * 32 + lane;
                // the key's scale (e4m3 inputs), applied after the head sum
                const float ks = F8 ? (s < L ? __ldg(k_scale + s) : 0.f) : 1.f;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    bool got = mbar_wait(&acc_full[a], acc_it[a] & 1, abort_flag, err,
                                         kDevTimeoutEpilogue);
                    got = __all_sync(0xffffffffu, got);
                    if (!got) {
                        ok = false;
                        break;
                    }
                    ++acc_it[a];
                    tc_fence_after();
                    const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16) +
                                           static_cast<uint32_t>(a * S::BN + cg * COLS);
                    const int tok_base = a * S::TOK_PER_ACC + cg * TOK_PER_HALF;
                    const float* wa = wW + a * COLS;
                    // 32-column chunks: chunk c + 1 is loaded while chunk c is
                    // scored.  Four partial sums per token (heads 0, 1, 2, 3
                    // mod 4) as two packed pairs; a token's score is stored as
                    // soon as its last head is in.
                    uint32_t buf[2][32];
                    tmem_ld32(taddr, buf[0]);
                    tmem_ld_wait();
                    uint64_t p01 = 0, p23 = 0;
#pragma unroll
                    for (int c = 0; c < NCHUNK; ++c) {
                        if (c < NCHUNK - 1) tmem_ld32(taddr + (c + 1) * 32, buf[(c + 1) & 1]);
                        const uint32_t(&v)[32] = buf[c & 1];
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const int col = c * 32 + j;
                            const ulonglong2 wv = *reinterpret_cast<const ulonglong2*>(wa + col);
                            p01 = f2_fma(wv.x, f2_pack(fmaxf(__uint_as_float(v[j]), 0.f),
                                                       fmaxf(__uint_as_float(v[j + 1]), 0.f)), p01);
                            p23 = f2_fma(wv.y, f2_pack(fmaxf(__uint_as_float(v[j + 2]), 0.f),
                                                       fmaxf(__uint_as_float(v[j + 3]), 0.f)), p23);
                            if ((col + 4) % H_I == 0) {
                                const float2 x = f2_unpack(p01), y = f2_unpack(p23);
                                const float sc = (x.x + x.y) + (y.x + y.y);
                                const int t = t0 + tok_base + col / H_I;
                                if (t < row_end && s <= t)
                                    scores[static_cast<long long>(t - row_begin) * ld + s] =
                                        F8 ? sc * ks : sc;
                                p01 = 0;
                                p23 = 0;
                            }
                        }
                        if (c < NCHUNK - 1) {
                            tmem_ld_wait();
                            if (c == NCHUNK - 2) {
                                // all of this accumulator is in registers: hand it back
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(&acc_empty[a]);
                            }
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int H_I, int NATOM, bool F8>
static int launch_prefill_t(ic_ctx* ctx, const void* qI, const void* kI, const void* w,
                            const float* q_scale, const float* k_scale, int L, int d_I,
                            int row_begin, int row_end, float* scores, int64_t ld, int q_row0,
                            int q_rows, cudaStream_t stream) {
    using S = PrefillShape<H_I, NATOM, F8>;
    auto kern = k_index_score_prefill<H_I, NATOM, F8>;
    static PerDeviceOnce attr_once;
    cudaError_t ea = attr_once.run(ctx->device, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
    });
    if (ea != cudaSuccess) return cuda_fail(ctx, ea, "cudaFuncSetAttribute(index_score)");
    CUtensorMap tm_q, tm_k;
    int rc;
    if (F8) {
        rc = make_tmap_u8_2d(ctx, &tm_q, qI, static_cast<uint64_t>(q_rows) * H_I, d_I, 128, S::BN,
                             true);
        if (rc) return rc;
        rc = make_tmap_u8_2d(ctx, &tm_k, kI, static_cast<uint64_t>(L), d_I, 128, S::BM, true);
    } else {
        rc = make_tmap_bf16_2d(ctx, &tm_q, qI, static_cast<uint64_t>(q_rows) * H_I, d_I, S::BN);
        if (rc) return rc;
        rc = make_tmap_bf16_2d(ctx, &tm_k, kI, static_cast<uint64_t>(L), d_I, S::BM);
    }
    if (rc) return rc;
    const int n_items = (row_end - row_begin + S::TQ - 1) / S::TQ;
    const int grid = n_items < ctx->num_sms ? n_items : ctx->num_sms;
    LaunchScope ls(ctx, IC_K_INDEX_SCORE, stream);
    kern<<<grid, S::THREADS, S::SMEM, stream>>>(tm_q, tm_k, static_cast<const __nv_bfloat16*>(w), q_scale,
                                         k_scale, scores, static_cast<long long>(ld), L, row_begin,
                                         row_end, n_items, q_row0, q_rows, ctx->dev_err);
    cudaError_t e = ls.done();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "index_score launch");
    return IC_OK;
}

int launch_index_score_prefill(ic_ctx* ctx, const void* qI, const void* kI, const void* w, int L,
                               int H_I, int d_I, int row_begin, int row_end, float* scores,
                               int64_t ld, cudaStream_t stream, int q_row0, int q_rows) {
    if (row_end <= row_begin) return IC_OK;
    if (q_rows < 0) q_rows = L;  // q_I and w hold every row
    const bool one_atom = d_I <= 64;
#define IC_PREFILL_CASE(H)                                                                      \
    case H:                                                                                     \
        return one_atom ? launch_prefill_t<H, 1, false>(ctx, qI, kI, w, nullptr, nullptr, L,    \
                                                        d_I, row_begin, row_end, scores, ld,    \
                                                        q_row0, q_rows, stream)                 \
                        : launch_prefill_t<H, 2, false>(ctx, qI, kI, w, nullptr, nullptr, L,    \
                                                        d_I, row_begin, row_end, scores, ld,    \
                                                        q_row0, q_rows, stream);
    switch (H_I) {
        IC_PREFILL_CASE(4)
        IC_PREFILL_CASE(8)
        IC_PREFILL_CASE(16)
        IC_PREFILL_CASE(32)
        IC_PREFILL_CASE(64)
        default:
            return fail(ctx, IC_ERR_UNSUPPORTED, "index_score: H_I=%d not in {4,8,16,32,64}", H_I);
    }
#undef IC_PREFILL_CASE
}

int launch_index_score_prefill_fp8(ic_ctx* ctx, const uint8_t* qI8, const float* q_scale,
                                   const uint8_t* kI8, const float* k_scale, const void* w, int L,
                                   int H_I, int d_I, int row_begin, int row_end, float* scores,
                                   int64_t ld, cudaStream_t stream) {
    if (row_end <= row_begin) return IC_OK;
    if (d_I != 128)
        return fail(ctx, IC_ERR_UNSUPPORTED, "index_score_fp8: d_I=%d (need 128)", d_I);
    switch (H_I) {
        case 16:
            return launch_prefill_t<16, 1, true>(ctx, qI8, kI8, w, q_scale, k_scale, L, d_I,
                                                 row_begin, row_end, scores, ld, 0, L, stream);
        case 32:
            return launch_prefill_t<32, 1, true>(ctx, qI8, kI8, w, q_scale, k_scale, L, d_I,
                                                 row_begin, row_end, scores, ld, 0, L, stream);
        case 64:
            return launch_prefill_t<64, 1, true>(ctx, qI8, kI8, w, q_scale, k_scale, L, d_I,
                                                 row_begin, row_end, scores, ld, 0, L, stream);
        default:
            return fail(ctx, IC_ERR_UNSUPPORTED, "index_score_fp8: H_I=%d not in {16,32,64}", H_I);
    }
}

}  // namespace ic
