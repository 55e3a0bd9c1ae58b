// C ABI of libindexcache (declared in include/indexcache.h): argument
// checking, the context (scratch, device error word, timing events),
// patterns, TMA descriptor encoding and the F/S layer loop.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "ic_internal.h"

namespace {
thread_local std::string g_last_error = "no error";
constexpr size_t kDefaultScratch = 2ull << 30;  // 2 GiB of fp32 score rows

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

namespace ic {

int fail(ic_ctx* ctx, int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    if (ctx)
        ctx->last_error = buf;
    else
        g_last_error = buf;
    return code;
}

int cuda_fail(ic_ctx* ctx, cudaError_t e, const char* what) {
    return fail(ctx, IC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int device_error(ic_ctx* ctx, int h) {
    if (h == kDevBadIndex)
        return fail(ctx, IC_ERR_DEVICE, "device: an index was outside [-1, kv_len)");
    if (h == kDevSmemMisaligned)
        return fail(ctx, IC_ERR_DEVICE, "device: dynamic shared memory not 1024-byte aligned");
    return fail(ctx, IC_ERR_TIMEOUT, "device: a bounded wait ran out (code %d)", h);
}

LaunchScope::LaunchScope(ic_ctx* c, int k, cudaStream_t s) : ctx(c), kernel(k), stream(s), slot(0) {
    if (!ctx->timing) return;
    if (ctx->pending == ctx->pool.size()) {
        ic_ctx::EventPair p{k, nullptr, nullptr};
        cudaEventCreate(&p.start);
        cudaEventCreate(&p.stop);
        ctx->pool.push_back(p);
    }
    slot = ctx->pending++;
    ctx->pool[slot].kernel = k;
    cudaEventRecord(ctx->pool[slot].start, stream);
}

cudaError_t LaunchScope::done() {
    cudaError_t e = cudaGetLastError();
    ctx->launch_count++;
    if (ctx->timing) cudaEventRecord(ctx->pool[slot].stop, stream);
    return e;
}

int ensure_buffer(ic_ctx* ctx, void** buf, size_t* cap, size_t bytes) {
    if (*cap >= bytes && *buf) return IC_OK;
    if (ctx->graphs_alive > 0)
        return fail(ctx, IC_ERR_NOMEM,
                    "scratch of %zu bytes needed while %d captured graph(s) hold the current "
                    "%zu-byte buffer; destroy them first",
                    bytes, ctx->graphs_alive, *cap);
    if (*buf) {
        cudaError_t e = cudaDeviceSynchronize();  // the old buffer may still be in use
        if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaDeviceSynchronize");
        cudaFree(*buf);
        *buf = nullptr;
        *cap = 0;
    }
    cudaError_t e = cudaMalloc(buf, bytes);
    if (e != cudaSuccess) {
        *buf = nullptr;
        cudaGetLastError();
        return fail(ctx, IC_ERR_NOMEM, "cudaMalloc(%zu bytes) failed: %s", bytes,
                    cudaGetErrorString(e));
    }
    *cap = bytes;
    return IC_OK;
}

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int make_tmap_bf16_2d(ic_ctx* ctx, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return fail(ctx, IC_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t gdim[2] = {cols, rows};
    const cuuint64_t gstride[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride,
                    box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(ctx, IC_ERR_CUDA, "cuTensorMapEncodeTiled(bf16 %llux%llu) failed: %d",
                    (unsigned long long)rows, (unsigned long long)cols, (int)r);
    return IC_OK;
}

int make_tmap_u8_2d(ic_ctx* ctx, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return fail(ctx, IC_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t gdim[2] = {cols, rows};
    const cuuint64_t gstride[1] = {cols};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), gdim, gstride,
                    box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(ctx, IC_ERR_CUDA, "cuTensorMapEncodeTiled(u8 %llux%llu) failed: %d",
                    (unsigned long long)rows, (unsigned long long)cols, (int)r);
    return IC_OK;
}

}  // namespace ic

using namespace ic;

static cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// ---------------------------------------------------------------- context
extern "C" int ic_version(void) { return 100; }

extern "C" int ic_ctx_create(ic_ctx** out, int device, size_t scratch_bytes) {
    if (!out) return fail(nullptr, IC_ERR_INVALID_ARG, "ic_ctx_create: out is NULL");
    *out = nullptr;
    cudaError_t e = cudaSetDevice(device);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "cudaSetDevice");
    ic_ctx* c = new ic_ctx();
    c->device = device;
    c->scratch_limit = scratch_bytes ? scratch_bytes : kDefaultScratch;
    e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device);
    if (e != cudaSuccess) {
        delete c;
        return cuda_fail(nullptr, e, "cudaDeviceGetAttribute");
    }
    e = cudaMalloc(&c->dev_err, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(c->dev_err, 0, sizeof(int));
    if (e != cudaSuccess) {
        delete c;
        return cuda_fail(nullptr, e, "ic_ctx_create: error word");
    }
    *out = c;
    return IC_OK;
}

extern "C" int ic_ctx_destroy(ic_ctx* ctx) {
    if (!ctx) return IC_ERR_INVALID_ARG;
    if (ctx->graphs_alive > 0)
        return fail(ctx, IC_ERR_INVALID_ARG, "ic_ctx_destroy: %d stack graph(s) still exist",
                    ctx->graphs_alive);
    cudaSetDevice(ctx->device);
    cudaDeviceSynchronize();
    cudaFree(ctx->scores);
    cudaFree(ctx->hist);
    cudaFree(ctx->dev_err);
    if (ctx->hs.ready) {
        for (int i = 0; i < ic_ctx::kHostSlots; ++i) {
            cudaFree(ctx->hs.slot[i]);
            cudaEventDestroy(ctx->hs.in_ready[i]);
            cudaEventDestroy(ctx->hs.computed[i]);
            cudaEventDestroy(ctx->hs.out_done[i]);
        }
        cudaStreamDestroy(ctx->hs.in);
        cudaStreamDestroy(ctx->hs.out);
    }
    if (ctx->ahead.ready) {
        cudaEventDestroy(ctx->ahead.start);
        for (int i = 0; i < 2; ++i) {
            cudaEventDestroy(ctx->ahead.indexed[i]);
            cudaEventDestroy(ctx->ahead.freed[i]);
        }
        cudaStreamDestroy(ctx->ahead.side);
    }
    for (auto& p : ctx->pool) {
        cudaEventDestroy(p.start);
        cudaEventDestroy(p.stop);
    }
    delete ctx;
    return IC_OK;
}

extern "C" const char* ic_last_error(const ic_ctx* ctx) {
    return ctx ? ctx->last_error.c_str() : g_last_error.c_str();
}

extern "C" int ic_sync_status(ic_ctx* ctx, void* stream) {
    if (!ctx) return IC_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(ctx, e, "ic_sync_status");
    int h = 0;
    e = cudaMemcpy(&h, ctx->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "ic_sync_status: read error word");
    if (h == 0) return IC_OK;
    cudaMemset(ctx->dev_err, 0, sizeof(int));
    return device_error(ctx, h);
}

extern "C" int ic_ctx_set_timing(ic_ctx* ctx, int enable) {
    if (!ctx) return IC_ERR_INVALID_ARG;
    ctx->timing = enable != 0;
    return IC_OK;
}

extern "C" int ic_ctx_get_timing(ic_ctx* ctx, int kernel, double* total_ms, int64_t* launches) {
    if (!ctx || kernel < 0 || kernel >= IC_K_COUNT)
        return fail(ctx, IC_ERR_INVALID_ARG, "ic_ctx_get_timing: bad kernel id");
    for (size_t i = 0; i < ctx->pending; ++i) {
        auto& p = ctx->pool[i];
        cudaError_t e = cudaEventSynchronize(p.stop);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaEventSynchronize");
        float ms = 0.f;
        cudaEventElapsedTime(&ms, p.start, p.stop);
        ctx->total_ms[p.kernel] += ms;
        ctx->launches[p.kernel] += 1;
    }
    ctx->pending = 0;
    if (total_ms) *total_ms = ctx->total_ms[kernel];
    if (launches) *launches = ctx->launches[kernel];
    return IC_OK;
}

extern "C" int ic_ctx_reset_timing(ic_ctx* ctx) {
    if (!ctx) return IC_ERR_INVALID_ARG;
    for (size_t i = 0; i < ctx->pending; ++i) cudaEventSynchronize(ctx->pool[i].stop);
    ctx->pending = 0;
    for (int k = 0; k < IC_K_COUNT; ++k) {
        ctx->total_ms[k] = 0;
        ctx->launches[k] = 0;
    }
    return IC_OK;
}

extern "C" int64_t ic_ctx_launch_count(const ic_ctx* ctx) { return ctx ? ctx->launch_count : -1; }

// ---------------------------------------------------------------- pattern
static int build_pattern(const std::string& c, ic_pattern** out) {
    if (c.empty()) return fail(nullptr, IC_ERR_PATTERN, "pattern: no layers");
    for (char ch : c)
        if (ch != 'F' && ch != 'S')
            return fail(nullptr, IC_ERR_PATTERN, "pattern: character '%c' is not F or S", ch);
    if (c[0] != 'F') return fail(nullptr, IC_ERR_PATTERN, "pattern: the first layer must be F");
    ic_pattern* p = new ic_pattern();
    p->c = c;
    p->src.resize(c.size());
    int last_f = 0;
    for (size_t l = 0; l < c.size(); ++l) {
        if (c[l] == 'F') last_f = static_cast<int>(l);
        p->src[l] = last_f;  // l itself for F, f(l) for S
    }
    *out = p;
    return IC_OK;
}

extern "C" int ic_create_pattern(const char* c, int n_layers, ic_pattern** out) {
    if (!c || !out || n_layers < 0)
        return fail(nullptr, IC_ERR_INVALID_ARG, "ic_create_pattern: bad arguments");
    *out = nullptr;
    return build_pattern(std::string(c, static_cast<size_t>(n_layers)), out);
}

extern "C" int ic_pattern_uniform(int n_layers, int r, ic_pattern** out) {
    if (!out || n_layers <= 0 || r <= 0)
        return fail(nullptr, IC_ERR_INVALID_ARG, "ic_pattern_uniform: bad arguments");
    std::string c(static_cast<size_t>(n_layers), 'S');
    for (int l = 0; l < n_layers; l += r) c[l] = 'F';
    return build_pattern(c, out);
}

extern "C" int ic_pattern_destroy(ic_pattern* p) {
    delete p;
    return IC_OK;
}

extern "C" int ic_pattern_size(const ic_pattern* p) { return p ? static_cast<int>(p->c.size()) : -1; }

extern "C" int ic_pattern_string(const ic_pattern* p, char* buf, int buflen) {
    if (!p || !buf || buflen < static_cast<int>(p->c.size()) + 1) return IC_ERR_INVALID_ARG;
    memcpy(buf, p->c.data(), p->c.size());
    buf[p->c.size()] = 0;
    return IC_OK;
}

extern "C" int ic_pattern_src(const ic_pattern* p, int32_t* src_out) {
    if (!p || !src_out) return IC_ERR_INVALID_ARG;
    memcpy(src_out, p->src.data(), p->src.size() * sizeof(int32_t));
    return IC_OK;
}

// ------------------------------------------------------- prefill indexer
static int check_index_args(ic_ctx* ctx, const void* qI, const void* kI, const void* w, int L,
                            int H_I, int d_I) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (!qI || !kI || !w) return fail(ctx, IC_ERR_INVALID_ARG, "index: NULL input");
    if (!aligned16(qI) || !aligned16(kI))
        return fail(ctx, IC_ERR_INVALID_ARG, "index: q_I and k_I must be 16-byte aligned");
    if (L <= 0) return fail(ctx, IC_ERR_SHAPE, "index: L=%d", L);
    if (H_I != 4 && H_I != 8 && H_I != 16 && H_I != 32 && H_I != 64)
        return fail(ctx, IC_ERR_UNSUPPORTED, "index: H_I=%d not in {4,8,16,32,64}", H_I);
    if (d_I != 32 && d_I != 64 && d_I != 128)
        return fail(ctx, IC_ERR_UNSUPPORTED, "index: d_I=%d not in {32,64,128}", d_I);
    if (static_cast<long long>(L) * H_I > (1ll << 31) - 1)
        return fail(ctx, IC_ERR_UNSUPPORTED, "index: L*H_I too large");
    return IC_OK;
}

extern "C" int ic_index_score(ic_ctx* ctx, const void* qI, const void* kI, const void* w, int L,
                              int H_I, int d_I, int row_begin, int row_end, float* scores,
                              int64_t ld, void* stream) {
    int rc = check_index_args(ctx, qI, kI, w, L, H_I, d_I);
    if (rc) return rc;
    if (!scores) return fail(ctx, IC_ERR_INVALID_ARG, "index_score: scores is NULL");
    if (row_begin < 0 || row_end > L || row_begin > row_end)
        return fail(ctx, IC_ERR_SHAPE, "index_score: rows [%d,%d) outside [0,%d)", row_begin,
                    row_end, L);
    if (ld < row_end || ld % 4 != 0)
        return fail(ctx, IC_ERR_SHAPE, "index_score: ld=%lld must be >= row_end and a multiple of 4",
                    (long long)ld);
    cudaSetDevice(ctx->device);
    return launch_index_score_prefill(ctx, qI, kI, w, L, H_I, d_I, row_begin, row_end, scores, ld,
                                      as_stream(stream));
}

extern "C" int ic_topk(ic_ctx* ctx, const float* scores, int64_t ld, int rows, int k,
                       int causal_base, const int32_t* row_len, int32_t* idx_out, int64_t ld_out,
                       void* stream) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (!idx_out || (!scores && rows > 0)) return fail(ctx, IC_ERR_INVALID_ARG, "topk: NULL pointer");
    if (rows < 0 || k < 1 || k > 2048 || ld_out < k || causal_base < 0)
        return fail(ctx, IC_ERR_SHAPE, "topk: rows=%d k=%d ld_out=%lld", rows, k, (long long)ld_out);
    if (ld % 4 != 0 || (reinterpret_cast<uintptr_t>(scores) & 15u))
        return fail(ctx, IC_ERR_INVALID_ARG, "topk: scores must be 16-byte aligned with ld %% 4 == 0");
    int max_len = 0;
    if (row_len) {
        max_len = static_cast<int>(ld);  // rows never exceed the row stride
    } else if (static_cast<long long>(causal_base) + rows > ld) {
        return fail(ctx, IC_ERR_SHAPE, "topk: causal rows exceed ld");
    }
    cudaSetDevice(ctx->device);
    return launch_topk(ctx, scores, ld, rows, k, causal_base, row_len, max_len, idx_out, ld_out,
                       as_stream(stream));
}

// F layer over query rows [r0, r1) (idx_out row 0 is row r0): rows t < k
// select {0..t} without scores; the other rows are scored in chunks whose
// fp32 rows fit in the scratch limit, each chunk followed by its top-k.
// `score(rb, re, scores, ld)` scores rows [rb, re).
template <class ScoreFn>
static int index_fp_range(ic_ctx* ctx, int r0, int r1, int k, int32_t* idx_out, cudaStream_t s,
                          ScoreFn score) {
    const int first = r0 > k ? r0 : (k < r1 ? k : r1);  // rows [r0, first) need no score
    if (first > r0) {
        int rc = launch_topk(ctx, nullptr, 0, first - r0, k, r0, nullptr, 0, idx_out, k, s);
        if (rc) return rc;
    }
    if (first >= r1) return IC_OK;
    const int64_t ld = (static_cast<int64_t>(r1) + 63) / 64 * 64;
    int64_t chunk = static_cast<int64_t>(ctx->scratch_limit / (static_cast<size_t>(ld) * 4));
    if (chunk < 1) return fail(ctx, IC_ERR_NOMEM, "index_fp: scratch too small for one row");
    if (chunk > r1 - first) chunk = r1 - first;
    int rc = ensure_buffer(ctx, reinterpret_cast<void**>(&ctx->scores), &ctx->scores_cap,
                           static_cast<size_t>(chunk) * ld * 4);
    if (rc) return rc;
    for (int rb = first; rb < r1; rb += static_cast<int>(chunk)) {
        const int re = static_cast<int>(rb + chunk < r1 ? rb + chunk : r1);
        const int64_t ldc = (static_cast<int64_t>(re) + 63) / 64 * 64;
        rc = score(rb, re, ctx->scores, ldc);
        if (rc) return rc;
        rc = launch_topk(ctx, ctx->scores, ldc, re - rb, k, rb,
                         nullptr, 0, idx_out + static_cast<int64_t>(rb - r0) * k, k, s);
        if (rc) return rc;
    }
    return IC_OK;
}

template <class ScoreFn>
static int index_fp_rows(ic_ctx* ctx, int L, int k, int32_t* idx_out, cudaStream_t s,
                         ScoreFn score) {
    return index_fp_range(ctx, 0, L, k, idx_out, s, score);
}

extern "C" int ic_index_fp(ic_ctx* ctx, const void* qI, const void* kI, const void* w, int L,
                           int H_I, int d_I, int k, int32_t* idx_out, void* stream) {
    int rc = check_index_args(ctx, qI, kI, w, L, H_I, d_I);
    if (rc) return rc;
    if (!idx_out) return fail(ctx, IC_ERR_INVALID_ARG, "index_fp: idx_out is NULL");
    if (k < 1 || k > 2048) return fail(ctx, IC_ERR_SHAPE, "index_fp: k=%d not in [1,2048]", k);
    cudaSetDevice(ctx->device);
    cudaStream_t s = as_stream(stream);
    return index_fp_rows(ctx, L, k, idx_out, s, [&](int rb, int re, float* sc, int64_t ldc) {
        return launch_index_score_prefill(ctx, qI, kI, w, L, H_I, d_I, rb, re, sc, ldc, s);
    });
}

// The F layer of one range of query rows whose q_I / w rows are held
// compactly (a rank's share of a prefill split across GPUs).
extern "C" int ic_index_fp_rows(ic_ctx* ctx, const void* qI_rows, const void* w_rows,
                                const void* kI, int L, int H_I, int d_I, int row_begin,
                                int row_end, int k, int32_t* idx_out, void* stream) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (k < 1 || k > 2048) return fail(ctx, IC_ERR_SHAPE, "index_fp_rows: k=%d not in [1,2048]", k);
    if (row_begin < 0 || row_end > L || row_begin > row_end)
        return fail(ctx, IC_ERR_SHAPE, "index_fp_rows: rows [%d,%d) outside [0,%d)", row_begin,
                    row_end, L);
    if (row_end == row_begin) return IC_OK;  // no rows: nothing is read or written
    int rc = check_index_args(ctx, qI_rows, kI, w_rows, L, H_I, d_I);
    if (rc) return rc;
    if (!idx_out) return fail(ctx, IC_ERR_INVALID_ARG, "index_fp_rows: idx_out is NULL");
    cudaSetDevice(ctx->device);
    cudaStream_t s = as_stream(stream);
    const int n = row_end - row_begin;
    return index_fp_range(ctx, row_begin, row_end, k, idx_out, s,
                          [&](int rb, int re, float* sc, int64_t ldc) {
                              return launch_index_score_prefill(ctx, qI_rows, kI, w_rows, L, H_I,
                                                                d_I, rb, re, sc, ldc, s, row_begin,
                                                                n);
                          });
}

// Causal-balanced split of L query rows over `world` ranks: 2*world chunks
// of near-equal size (the first L % (2*world) one row longer); rank r takes
// chunks r and 2*world - 1 - r, so an early (cheap) and a late (costly)
// chunk pair up.
extern "C" int ic_prefill_partition(int L, int world, int rank, int32_t* ranges, int* n_ranges) {
    if (!ranges || !n_ranges || L < 0 || world < 1 || rank < 0 || rank >= world)
        return fail(nullptr, IC_ERR_INVALID_ARG, "prefill_partition: L=%d world=%d rank=%d", L,
                    world, rank);
    const int64_t nch = 2ll * world;
    auto start = [&](int64_t c) {  // first row of chunk c
        const int64_t base = L / nch, extra = L % nch;
        return c * base + (c < extra ? c : extra);
    };
    const int64_t ca = rank, cb = nch - 1 - rank;
    ranges[0] = static_cast<int32_t>(start(ca));
    ranges[1] = static_cast<int32_t>(start(ca + 1));
    ranges[2] = static_cast<int32_t>(start(cb));
    ranges[3] = static_cast<int32_t>(start(cb + 1));
    *n_ranges = 2;
    return IC_OK;
}

// ------------------------------------------------ FP8 prefill indexer
static int check_index_fp8_args(ic_ctx* ctx, const uint8_t* qI8, const float* q_scale,
                                const uint8_t* kI8, const float* k_scale, const void* w, int L,
                                int H_I, int d_I) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (!qI8 || !q_scale || !kI8 || !k_scale || !w)
        return fail(ctx, IC_ERR_INVALID_ARG, "index_fp8: NULL input");
    if (!aligned16(qI8) || !aligned16(kI8))
        return fail(ctx, IC_ERR_INVALID_ARG, "index_fp8: qI8 and kI8 must be 16-byte aligned");
    if (L < 1 || L > (1 << 24)) return fail(ctx, IC_ERR_SHAPE, "index_fp8: L=%d", L);
    if (d_I != 128 || (H_I != 16 && H_I != 32 && H_I != 64))
        return fail(ctx, IC_ERR_UNSUPPORTED, "index_fp8: H_I=%d d_I=%d (need {16,32,64}, 128)",
                    H_I, d_I);
    return IC_OK;
}

extern "C" int ic_index_score_fp8(ic_ctx* ctx, const uint8_t* qI8, const float* q_scale,
                                  const uint8_t* kI8, const float* k_scale, const void* w, int L,
                                  int H_I, int d_I, int row_begin, int row_end, float* scores,
                                  int64_t ld, void* stream) {
    int rc = check_index_fp8_args(ctx, qI8, q_scale, kI8, k_scale, w, L, H_I, d_I);
    if (rc) return rc;
    if (!scores) return fail(ctx, IC_ERR_INVALID_ARG, "index_score_fp8: scores is NULL");
    if (row_begin < 0 || row_end > L || row_begin > row_end)
        return fail(ctx, IC_ERR_SHAPE, "index_score_fp8: rows [%d,%d) outside [0,%d)", row_begin,
                    row_end, L);
    if (ld < row_end || ld % 4 != 0)
        return fail(ctx, IC_ERR_SHAPE,
                    "index_score_fp8: ld=%lld must be >= row_end and a multiple of 4",
                    (long long)ld);
    cudaSetDevice(ctx->device);
    return launch_index_score_prefill_fp8(ctx, qI8, q_scale, kI8, k_scale, w, L, H_I, d_I,
                                          row_begin, row_end, scores, ld, as_stream(stream));
}

extern "C" int ic_index_fp_fp8(ic_ctx* ctx, const uint8_t* qI8, const float* q_scale,
                               const uint8_t* kI8, const float* k_scale, const void* w, int L,
                               int H_I, int d_I, int k, int32_t* idx_out, void* stream) {
    int rc = check_index_fp8_args(ctx, qI8, q_scale, kI8, k_scale, w, L, H_I, d_I);
    if (rc) return rc;
    if (!idx_out) return fail(ctx, IC_ERR_INVALID_ARG, "index_fp_fp8: idx_out is NULL");
    if (k < 1 || k > 2048) return fail(ctx, IC_ERR_SHAPE, "index_fp_fp8: k=%d not in [1,2048]", k);
    cudaSetDevice(ctx->device);
    cudaStream_t s = as_stream(stream);
    return index_fp_rows(ctx, L, k, idx_out, s, [&](int rb, int re, float* sc, int64_t ldc) {
        return launch_index_score_prefill_fp8(ctx, qI8, q_scale, kI8, k_scale, w, L, H_I, d_I, rb,
                                              re, sc, ldc, s);
    });
}

extern "C" int ic_index_reuse(const int32_t* idx_cache, const int32_t** idx_out) {
    if (!idx_cache || !idx_out) return fail(nullptr, IC_ERR_INVALID_ARG, "index_reuse: NULL");
    *idx_out = idx_cache;
    return IC_OK;
}

// -------------------------------------------------------- decode indexer
static int check_decode_args(ic_ctx* ctx, const void* q, const void* w, const uint8_t* kI8,
                             const float* kI_scale, const int32_t* seq_len, int B, int S_max,
                             int H_I, int d_I) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (!q || !w || !kI8 || !kI_scale || !seq_len)
        return fail(ctx, IC_ERR_INVALID_ARG, "decode index: NULL input");
    if (!aligned16(q) || !aligned16(kI8))
        return fail(ctx, IC_ERR_INVALID_ARG, "decode index: q and kI8 must be 16-byte aligned");
    if (B <= 0 || S_max <= 0) return fail(ctx, IC_ERR_SHAPE, "decode index: B=%d S_max=%d", B, S_max);
    if ((H_I != 32 && H_I != 64) || d_I != 128)
        return fail(ctx, IC_ERR_UNSUPPORTED, "decode index: H_I=%d d_I=%d (need {32,64}, 128)", H_I,
                    d_I);
    return IC_OK;
}

extern "C" int ic_index_score_decode(ic_ctx* ctx, const void* q, const void* w, const uint8_t* kI8,
                                     const float* kI_scale, const int32_t* seq_len, int B,
                                     int S_max, int H_I, int d_I, float* scores, int64_t ld,
                                     void* stream) {
    int rc = check_decode_args(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, H_I, d_I);
    if (rc) return rc;
    if (!scores) return fail(ctx, IC_ERR_INVALID_ARG, "decode index: scores is NULL");
    if (ld < S_max || ld % 4 != 0)
        return fail(ctx, IC_ERR_SHAPE, "decode index: ld=%lld", (long long)ld);
    cudaSetDevice(ctx->device);
    return launch_index_score_decode(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, H_I, d_I, scores,
                                     ld, as_stream(stream));
}

extern "C" int ic_index_fp_decode(ic_ctx* ctx, const void* q, const void* w, const uint8_t* kI8,
                                  const float* kI_scale, const int32_t* seq_len, int B, int S_max,
                                  int H_I, int d_I, int k, int32_t* idx_out, void* stream) {
    int rc = check_decode_args(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, H_I, d_I);
    if (rc) return rc;
    if (!idx_out) return fail(ctx, IC_ERR_INVALID_ARG, "decode index: idx_out is NULL");
    if (k < 1 || k > 2048) return fail(ctx, IC_ERR_SHAPE, "decode index: k=%d", k);
    cudaSetDevice(ctx->device);
    const int64_t ld = (static_cast<int64_t>(S_max) + 63) / 64 * 64;
    rc = ensure_buffer(ctx, reinterpret_cast<void**>(&ctx->scores), &ctx->scores_cap,
                       static_cast<size_t>(B) * ld * 4);
    if (rc) return rc;
    cudaStream_t s = as_stream(stream);
    // When the top-k takes the cluster form, the scan also counts each
    // sequence's scores by the top-k's first radix digit, so the top-k knows
    // its threshold bin before it reads a score.
    uint32_t* hist = nullptr;
    if (topk_uses_cluster(ctx, B, true, S_max)) {
        const size_t bytes = static_cast<size_t>(B) * 2048 * sizeof(uint32_t);
        if (ctx->hist_cap < bytes || ctx->hist == nullptr) {
            rc = ensure_buffer(ctx, reinterpret_cast<void**>(&ctx->hist), &ctx->hist_cap, bytes);
            if (rc) return rc;
            ctx->hist_dirty = true;
        }
        if (ctx->hist_dirty) {
            cudaError_t e = cudaMemsetAsync(ctx->hist, 0, ctx->hist_cap, s);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "decode index: clear histograms");
            ctx->hist_dirty = false;
        }
        hist = ctx->hist;
    }
    if (hist) ctx->hist_dirty = true;  // until the top-k that clears it is enqueued
    rc = launch_index_score_decode(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, H_I, d_I,
                                   ctx->scores, ld, s, hist);
    if (rc) return rc;
    rc = launch_topk(ctx, ctx->scores, ld, B, k, 0, seq_len, S_max, idx_out, k, s, hist);
    if (rc == IC_OK) ctx->hist_dirty = false;
    return rc;
}

// ------------------------------------------------------ sparse attention
extern "C" int ic_sparse_attn(ic_ctx* ctx, const void* Q, const void* K, const void* V,
                              const int32_t* idx, int rows, int Hq, int d, int k, int rows_per_seq,
                              int64_t kv_seq_stride, int kv_len, float scale, void* out,
                              void* stream) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (rows < 0 || k < 1 || k > 2048 || Hq < 1 || Hq > 16 || kv_len < 0 || rows_per_seq < 0 ||
        kv_seq_stride < 0)
        return fail(ctx, IC_ERR_SHAPE, "sparse_attn: rows=%d Hq=%d k=%d kv_len=%d", rows, Hq, k,
                    kv_len);
    if (d != 64 && d != 128) return fail(ctx, IC_ERR_UNSUPPORTED, "sparse_attn: d=%d", d);
    if (kv_len > (1 << 24))
        return fail(ctx, IC_ERR_UNSUPPORTED, "sparse_attn: kv_len=%d above 2^24", kv_len);
    if (rows == 0) return IC_OK;
    if (!Q || !K || !V || !idx || !out) return fail(ctx, IC_ERR_INVALID_ARG, "sparse_attn: NULL");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || (reinterpret_cast<uintptr_t>(out) & 7u))
        return fail(ctx, IC_ERR_INVALID_ARG,
                    "sparse_attn: Q, K, V must be 16-byte and out 8-byte aligned");
    if (scale <= 0.f) scale = 1.0f / sqrtf(static_cast<float>(d));
    cudaSetDevice(ctx->device);
    return launch_sparse_attn(ctx, Q, K, V, idx, rows, Hq, d, k, rows_per_seq, kv_seq_stride,
                              kv_len, scale, out, as_stream(stream));
}

// -------------------------------------------------- cross-layer overlap
extern "C" int ic_index_overlap(ic_ctx* ctx, const int32_t* idx_a, const int32_t* idx_b, int rows,
                                int k, int n_keys, int32_t* hits, void* stream) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (rows < 0 || k < 1 || n_keys < 1)
        return fail(ctx, IC_ERR_SHAPE, "index_overlap: rows=%d k=%d n_keys=%d", rows, k, n_keys);
    if (rows == 0) return IC_OK;
    if (!idx_a || !idx_b || !hits) return fail(ctx, IC_ERR_INVALID_ARG, "index_overlap: NULL");
    cudaSetDevice(ctx->device);
    return launch_index_overlap(ctx, idx_a, idx_b, rows, k, n_keys, hits, as_stream(stream));
}

// ------------------------------------------------------------ layer stack
namespace ic {
// One layer of the stack ([IC] Figure 2): an F layer runs the indexer and
// top-k into idx_cache, an S layer reuses it; then the layer's attention.
int run_stack_layer(ic_ctx* ctx, char c, const ic_layer_io& io, const ic_layer_io* next,
                    const ic_stack_dims* dims, int32_t* idx_cache, void* stream) {
    const bool prefill = dims->mode == IC_PREFILL;
    const int rows = prefill ? dims->L : dims->B;
    const int k = dims->k;
    // Decode layers of a small batch are short and leave most SMs idle: each
    // kernel is launched as a programmatic dependent of the previous one, so
    // it starts during that kernel's tail.  Every kernel waits for its
    // predecessor before reading what a previous layer (or its own F-layer
    // top-k) produces: the query inputs, the newest K/V row, the index cache
    // of an F layer.  An S layer's attention reads the index cache (written by
    // an earlier F layer) and warms L2 with the cached K/V rows at those
    // slots before it waits.  Used while the split attention of every row
    // fits one CTA per SM (B * 8 <= SMs); with a fuller GPU the early
    // dependents slowed the step (measured: B = 32 x 16 layers 0.54 ->
    // 0.60 ms, B = 8 x 47 layers 1.29 -> 1.24 ms).
    const bool pdl = !prefill && static_cast<long long>(dims->B) * 8 <= ctx->num_sms;
    struct PdlScope {
        ic_ctx* c;
        ~PdlScope() {
            c->pdl = 0;
            c->pf_K = c->pf_V = nullptr;
        }
    } pdl_scope{ctx};
    int rc;
    if (c == 'F') {
        ctx->pdl = pdl ? 1 : 0;
        if (prefill)
            rc = ic_index_fp(ctx, io.qI, io.kI, io.w, dims->L, dims->H_I, dims->d_I, k, idx_cache,
                             stream);
        else
            rc = ic_index_fp_decode(ctx, io.qI, io.w, io.kI8, io.kI_scale, dims->seq_len, dims->B,
                                    dims->S_max, dims->H_I, dims->d_I, k, idx_cache, stream);
        if (rc) return rc;
    }
    // S layer: the cache is used as it stands (no kernel)
    ctx->pdl = !pdl ? 0 : (c == 'F' ? 1 : 2);
    const int32_t* idx = nullptr;
    ic_index_reuse(idx_cache, &idx);
    if (io.idx_snapshot) {
        cudaError_t e = cudaMemcpyAsync(io.idx_snapshot, idx,
                                        static_cast<size_t>(rows) * k * sizeof(int32_t),
                                        cudaMemcpyDeviceToDevice, as_stream(stream));
        if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack: snapshot copy");
    }
    if (prefill)
        return ic_sparse_attn(ctx, io.Q, io.K, io.V, idx, rows, dims->Hq, dims->d, k, 0, 0, dims->L,
                              dims->scale, io.out, stream);
    // Decode: the next S layer gathers its own K/V at these same slots.  Its
    // cached rows are already in HBM, so this layer's CTAs warm L2 with them
    // after their own gather, overlapping that traffic with this layer's merge
    // and the launch in between.  (Small batches already do this in the S
    // layer itself, before its programmatic wait.)
    if (next && !pdl) {
        ctx->pf_K = next->K;
        ctx->pf_V = next->V;
    }
    return ic_sparse_attn(ctx, io.Q, io.K, io.V, idx, rows, dims->Hq, dims->d, k, 1,
                          static_cast<int64_t>(dims->S_max) * dims->d, dims->S_max, dims->scale,
                          io.out, stream);
}

int check_stack_args(ic_ctx* ctx, const ic_pattern* pattern, const void* layers,
                     const ic_stack_dims* dims, const int32_t* idx_cache) {
    if (!ctx) return fail(nullptr, IC_ERR_INVALID_ARG, "context is NULL");
    if (!pattern || !layers || !dims || !idx_cache)
        return fail(ctx, IC_ERR_INVALID_ARG, "run_stack: NULL argument");
    if (dims->mode != IC_PREFILL && dims->mode != IC_DECODE)
        return fail(ctx, IC_ERR_INVALID_ARG, "run_stack: mode %d", dims->mode);
    return IC_OK;
}
}  // namespace ic

extern "C" int ic_run_stack_rows(ic_ctx* ctx, const ic_pattern* pattern, const ic_layer_io* layers,
                                 const ic_stack_dims* dims, const int32_t* ranges, int n_ranges,
                                 int32_t* idx_cache, void* stream) {
    int rc = check_stack_args(ctx, pattern, layers, dims, idx_cache);
    if (rc) return rc;
    if (dims->mode != IC_PREFILL)
        return fail(ctx, IC_ERR_INVALID_ARG, "run_stack_rows: prefill stacks only");
    if (!ranges || n_ranges < 1) return fail(ctx, IC_ERR_INVALID_ARG, "run_stack_rows: no ranges");
    int64_t rows = 0;
    for (int i = 0; i < n_ranges; ++i) {
        const int a = ranges[2 * i], b = ranges[2 * i + 1];
        if (a < 0 || b > dims->L || a > b)
            return fail(ctx, IC_ERR_SHAPE, "run_stack_rows: range [%d,%d) outside [0,%d)", a, b,
                        dims->L);
        rows += b - a;
    }
    cudaSetDevice(ctx->device);
    const int N = static_cast<int>(pattern->c.size());
    const int k = dims->k;
    for (int l = 0; l < N; ++l) {
        const ic_layer_io& io = layers[l];
        if (pattern->c[l] == 'F') {
            int64_t off = 0;
            for (int i = 0; i < n_ranges; ++i) {
                const int a = ranges[2 * i], b = ranges[2 * i + 1];
                const char* q = static_cast<const char*>(io.qI) + off * dims->H_I * dims->d_I * 2;
                const char* w = static_cast<const char*>(io.w) + off * dims->H_I * 2;
                rc = ic_index_fp_rows(ctx, q, w, io.kI, dims->L, dims->H_I, dims->d_I, a, b, k,
                                      idx_cache + off * k, stream);
                if (rc) return rc;
                off += b - a;
            }
        }
        const int32_t* idx = nullptr;
        ic_index_reuse(idx_cache, &idx);
        if (io.idx_snapshot) {
            cudaError_t e = cudaMemcpyAsync(io.idx_snapshot, idx,
                                            static_cast<size_t>(rows) * k * sizeof(int32_t),
                                            cudaMemcpyDeviceToDevice, as_stream(stream));
            if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_rows: snapshot copy");
        }
        rc = ic_sparse_attn(ctx, io.Q, io.K, io.V, idx, static_cast<int>(rows), dims->Hq, dims->d,
                            k, 0, 0, dims->L, dims->scale, io.out, stream);
        if (rc) return rc;
    }
    return IC_OK;
}

extern "C" int ic_run_stack(ic_ctx* ctx, const ic_pattern* pattern, const ic_layer_io* layers,
                            const ic_stack_dims* dims, int32_t* idx_cache, void* stream) {
    int rc = check_stack_args(ctx, pattern, layers, dims, idx_cache);
    if (rc) return rc;
    cudaSetDevice(ctx->device);
    const int N = static_cast<int>(pattern->c.size());
    for (int l = 0; l < N; ++l) {
        const ic_layer_io* next = l + 1 < N && pattern->c[l + 1] == 'S' ? &layers[l + 1] : nullptr;
        rc = run_stack_layer(ctx, pattern->c[l], layers[l], next, dims, idx_cache, stream);
        if (rc) return rc;
    }
    return IC_OK;
}
