// Host-side internals of libindexcache: the context and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "ic_errors.h"
#include "indexcache.h"

struct ic_ctx {
    int device = 0;
    int num_sms = 148;
    size_t scratch_limit = 0;       // bound on the prefill score scratch (bytes)
    float* scores = nullptr;        // score scratch (fp32 rows)
    size_t scores_cap = 0;          // bytes
    // decode: per-sequence first-digit histograms of the scores ([B][2048]
    // uint32), written by the scan and read (then cleared) by the cluster
    // top-k; zero between uses, `hist_dirty` when a use may have stopped
    // between the two launches
    uint32_t* hist = nullptr;
    size_t hist_cap = 0;            // bytes
    bool hist_dirty = false;
    int* dev_err = nullptr;         // device error word (first error wins)
    std::string last_error;
    bool timing = false;
    struct EventPair {
        int kernel;
        cudaEvent_t start, stop;
    };
    std::vector<EventPair> pool;    // reusable event pairs
    size_t pending = 0;             // pairs recorded since the last harvest
    double total_ms[IC_K_COUNT] = {0};
    int64_t launches[IC_K_COUNT] = {0};
    int64_t launch_count = 0;
    int graphs_alive = 0;           // captured stack graphs that use this context's buffers
    // Programmatic dependent launch, set by the decode stack around its own
    // launches: 0 off; 1 the kernel may start while the previous kernel in the
    // stream finishes and waits for it before reading anything; 2 (attention
    // of an S layer) it may also read the index cache and warm L2 with the
    // K/V rows it will gather before that wait.
    int pdl = 0;
    // set by the decode stack for one attention launch: the next layer's K/V
    // (an S layer, which reuses this layer's index slots), whose rows at those
    // slots the attention kernel prefetches into L2 once its own gather is done
    const void* pf_K = nullptr;
    const void* pf_V = nullptr;
    // ic_run_stack_host: kHostSlots device staging slots, a copy-in and a
    // copy-out stream, and per-slot events (created on first use)
    static constexpr int kHostSlots = 4;
    struct HostStack {
        bool ready = false;
        cudaStream_t in = nullptr, out = nullptr;
        cudaEvent_t in_ready[kHostSlots] = {}, computed[kHostSlots] = {}, out_done[kHostSlots] = {};
        void* slot[kHostSlots] = {};
        size_t slot_cap = 0;  // bytes per slot
    } hs;
    // ic_run_stack_ahead: the side stream that runs the F layers' indexers,
    // and its fork and buffer events (created on first use)
    struct Ahead {
        bool ready = false;
        cudaStream_t side = nullptr;
        cudaEvent_t start = nullptr, indexed[2] = {}, freed[2] = {};
    } ahead;
};

struct ic_pattern {
    std::string c;
    std::vector<int32_t> src;
};

namespace ic {

constexpr int kMaxDevices = 64;

// Once-per-device set-up for host state that CUDA keeps per device, such as
// a kernel's maximum dynamic shared memory (cudaFuncSetAttribute acts on the
// current device only).  run(device, f) calls f() the first time it is asked
// for `device`, and again after f() failed; it is safe to call from several
// host threads at once.  Devices past kMaxDevices run f() on every call.
class PerDeviceOnce {
  public:
    template <class F>
    cudaError_t run(int device, F&& f) {
        if (device < 0 || device >= kMaxDevices) return f();
        const uint64_t bit = 1ull << device;
        if (done_.load(std::memory_order_acquire) & bit) return cudaSuccess;
        std::lock_guard<std::mutex> lock(m_);
        if (done_.load(std::memory_order_relaxed) & bit) return cudaSuccess;
        const cudaError_t e = f();
        if (e == cudaSuccess) done_.fetch_or(bit, std::memory_order_release);
        return e;
    }

  private:
    std::atomic<uint64_t> done_{0};
    std::mutex m_;
};

// Records the message on ctx (or the global slot) and returns code.
int fail(ic_ctx* ctx, int code, const char* fmt, ...);
int cuda_fail(ic_ctx* ctx, cudaError_t e, const char* what);
// Maps a nonzero device error word to its IC_ERR_* code and message.
int device_error(ic_ctx* ctx, int h);

// Brackets one kernel launch with timing events when timing is enabled and
// counts it.  Usage: LaunchScope ls(ctx, IC_K_TOPK, stream); kernel<<<>>>; ls.done();
// Appends the programmatic-dependent-launch attribute to attrs[n] when the
// context asks for it (ctx->pdl != 0).
inline void add_pdl_attr(const ic_ctx* ctx, cudaLaunchAttribute* attrs, unsigned int& n) {
    if (!ctx->pdl) return;
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
}

struct LaunchScope {
    ic_ctx* ctx;
    int kernel;
    cudaStream_t stream;
    size_t slot;
    LaunchScope(ic_ctx* c, int k, cudaStream_t s);
    cudaError_t done();
};

// Grows a scratch buffer to at least `bytes`.  Returns IC_OK / IC_ERR_NOMEM.
int ensure_buffer(ic_ctx* ctx, void** buf, size_t* cap, size_t bytes);

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// 2-D bf16 tensor map over [rows, cols] (cols contiguous) with a
// box of {64 columns, box_rows rows} and the 128-byte swizzle.
int make_tmap_bf16_2d(ic_ctx* ctx, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows);
// Same for an 8-bit tensor, box {box_cols columns, box_rows rows}, with the
// 128-byte swizzle (box_cols = 128) or none.
int make_tmap_u8_2d(ic_ctx* ctx, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_cols, uint32_t box_rows, bool swizzle128);

// ----------------------------------------------------------------- launchers
// One layer of the F/S stack (shared by ic_run_stack and ic_run_stack_host).
// `next` is the following layer when it is an S layer whose K/V are in device
// memory (it reuses this layer's index slots), else null.
int run_stack_layer(ic_ctx* ctx, char c, const ic_layer_io& io, const ic_layer_io* next,
                    const ic_stack_dims* dims, int32_t* idx_cache, void* stream);
int check_stack_args(ic_ctx* ctx, const ic_pattern* pattern, const void* layers,
                     const ic_stack_dims* dims, const int32_t* idx_cache);

// q_I and w hold rows [q_row0, q_row0 + q_rows) (q_rows < 0: every row of L)
int launch_index_score_prefill(ic_ctx* ctx, const void* qI, const void* kI, const void* w, int L,
                               int H_I, int d_I, int row_begin, int row_end, float* scores,
                               int64_t ld, cudaStream_t stream, int q_row0 = 0, int q_rows = -1);
// hist (optional, zero on entry): [B][2048] counts of the written scores
// by the top 11 bits of their order key, for launch_topk
int launch_index_score_decode(ic_ctx* ctx, const void* q, const void* w, const uint8_t* kI8,
                              const float* kI_scale, const int32_t* seq_len, int B, int S_max,
                              int H_I, int d_I, float* scores, int64_t ld, cudaStream_t stream,
                              uint32_t* hist = nullptr);
// Whether launch_topk takes the cluster form (a thread-block cluster per row)
// for these rows; only that form uses a precomputed histogram.
bool topk_uses_cluster(const ic_ctx* ctx, int rows, bool has_row_len, int max_len);
// hist (optional, cluster form only): the rows' first-digit histograms from
// launch_index_score_decode; read, then cleared to zero for the next use
int launch_topk(ic_ctx* ctx, const float* scores, int64_t ld, int rows, int k, int causal_base,
                const int32_t* row_len, int max_len, int32_t* idx_out, int64_t ld_out,
                cudaStream_t stream, uint32_t* hist = nullptr);
int launch_index_score_prefill_fp8(ic_ctx* ctx, const uint8_t* qI8, const float* q_scale,
                                   const uint8_t* kI8, const float* k_scale, const void* w, int L,
                                   int H_I, int d_I, int row_begin, int row_end, float* scores,
                                   int64_t ld, cudaStream_t stream);
int launch_index_overlap(ic_ctx* ctx, const int32_t* a, const int32_t* b, int rows, int k,
                         int n_keys, int32_t* hits, cudaStream_t stream);
int launch_sparse_attn(ic_ctx* ctx, const void* Q, const void* K, const void* V,
                       const int32_t* idx, int rows, int Hq, int d, int k, int rows_per_seq,
                       int64_t kv_seq_stride, int kv_len, float scale, void* out,
                       cudaStream_t stream);

}  // namespace ic
