// ic_index_fp_decode_noalloc: the decode F-layer indexer (FP8 key scan +
// per-sequence top-k) for callers that cannot allocate device memory.
//
// Who needs it: serving engines that hand all free HBM to their own KV-cache
// pool and forbid cudaMalloc on the decode path (the call may fail for lack
// of memory, and it synchronizes the device, which stalls a latency-bound
// per-token loop), and callers replaying the decode step in a captured
// stream, where an allocation cannot be issued.  The regular
// ic_index_fp_decode grows its context's scratch with cudaMalloc when the
// score rows do not fit.
//
// This variant keeps its fp32 score rows in a fixed array in device global
// memory, defined below, and needs no context.  The array is part of the
// library's module, so every GPU that loads the library holds it
// (kNoAllocScoreFloats fp32 scores) until the process exits.  Every call
// shares it: calls whose kernels overlap on the GPU (different streams, no
// ordering) race on it.  No entry of the array needs to start at any
// particular value: the scan writes every score the top-k reads.
//
// Errors found on the device (a bounded wait that ran out, a misaligned
// shared-memory window) are latched in a device word of the same kind;
// ic_noalloc_sync_status reads and clears it without allocating.  The host
// side of each call holds a per-device lock, so calls from several host
// threads are safe on the host (their kernels still share the array).
#include <string.h>

#include <mutex>

#include "ic_internal.h"

namespace {

// 4 Mi fp32 scores = 16 MiB: B * round_up(S_max, 64) must not exceed this.
constexpr size_t kNoAllocScoreFloats = size_t(4) << 20;
using ic::kMaxDevices;

}  // namespace

// Scratch for the score rows and the device error word.  In host code these
// names are host-side stand-ins, not device addresses: the set-up below asks
// the runtime for the device address before any kernel gets one.
static __device__ __align__(256) float g_noalloc_scores[kNoAllocScoreFloats];
static __device__ __align__(256) int g_noalloc_err[64];

namespace {

struct NoAllocDevice {
    std::mutex lock;  // held for the host side of every call on this device
    bool ready = false;
    ic_ctx ctx;  // host-side view; its pointers alias the static arrays above
};
NoAllocDevice g_dev[kMaxDevices];

// Once per device, with that device current and its lock held: resolve the
// device addresses of the static arrays and fill a context that points at
// them.
int setup_device(int device, ic_ctx** out) {
    NoAllocDevice& d = g_dev[device];
    if (!d.ready) {
        void* scores = nullptr;
        void* err = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&scores, g_noalloc_scores);
        if (e != cudaSuccess)
            return ic::fail(nullptr, IC_ERR_CUDA, "noalloc set-up: cudaGetSymbolAddress(scores): %s",
                            cudaGetErrorString(e));
        e = cudaGetSymbolAddress(&err, g_noalloc_err);
        if (e != cudaSuccess)
            return ic::fail(nullptr, IC_ERR_CUDA, "noalloc set-up: cudaGetSymbolAddress(err): %s",
                            cudaGetErrorString(e));
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
        if (e != cudaSuccess)
            return ic::fail(nullptr, IC_ERR_CUDA, "noalloc set-up: SM count: %s",
                            cudaGetErrorString(e));
        d.ctx.device = device;
        d.ctx.num_sms = sms;
        d.ctx.scores = static_cast<float*>(scores);
        d.ctx.scores_cap = kNoAllocScoreFloats * sizeof(float);
        d.ctx.dev_err = static_cast<int*>(err);
        d.ctx.timing = false;
        d.ready = true;
    }
    *out = &d.ctx;
    return IC_OK;
}

}  // namespace

extern "C" int ic_index_fp_decode_noalloc(const void* q, const void* w, const uint8_t* kI8,
                                          const float* kI_scale, const int32_t* seq_len, int B,
                                          int S_max, int H_I, int d_I, int k, int32_t* idx_out,
                                          void* stream) {
    if (!q || !w || !kI8 || !kI_scale || !seq_len || !idx_out)
        return ic::fail(nullptr, IC_ERR_INVALID_ARG, "decode noalloc: NULL pointer");
    if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(kI8) & 15u))
        return ic::fail(nullptr, IC_ERR_INVALID_ARG,
                        "decode noalloc: q and kI8 must be 16-byte aligned");
    if (B <= 0 || S_max <= 0 || k < 1 || k > 2048)
        return ic::fail(nullptr, IC_ERR_SHAPE, "decode noalloc: B=%d S_max=%d k=%d", B, S_max, k);
    if ((H_I != 32 && H_I != 64) || d_I != 128)
        return ic::fail(nullptr, IC_ERR_UNSUPPORTED, "decode noalloc: H_I=%d d_I=%d", H_I, d_I);
    const int64_t ld = (static_cast<int64_t>(S_max) + 63) / 64 * 64;
    if (static_cast<uint64_t>(B) * static_cast<uint64_t>(ld) > kNoAllocScoreFloats)
        return ic::fail(nullptr, IC_ERR_UNSUPPORTED,
                        "decode noalloc: B * round_up(S_max, 64) = %lld scores exceeds the fixed "
                        "scratch of %zu scores (16 MiB); use ic_index_fp_decode",
                        static_cast<long long>(B) * ld, kNoAllocScoreFloats);
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess || device < 0 || device >= kMaxDevices)
        return ic::fail(nullptr, IC_ERR_CUDA, "decode noalloc: no current device");
    std::lock_guard<std::mutex> lock(g_dev[device].lock);
    ic_ctx* ctx = nullptr;
    int rc = setup_device(device, &ctx);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = ic::launch_index_score_decode(ctx, q, w, kI8, kI_scale, seq_len, B, S_max, H_I, d_I,
                                       ctx->scores, ld, s);
    if (rc == IC_OK)
        rc = ic::launch_topk(ctx, ctx->scores, ld, B, k, 0, seq_len, S_max, idx_out, k, s);
    if (rc) ic::fail(nullptr, rc, "%s", ctx->last_error.c_str());
    return rc;
}

extern "C" int ic_noalloc_sync_status(void* stream) {
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess || device < 0 || device >= kMaxDevices)
        return ic::fail(nullptr, IC_ERR_CUDA, "noalloc status: no current device");
    e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return ic::cuda_fail(nullptr, e, "noalloc status: stream");
    // copies between the symbol and a host int: no device allocation
    int h = 0;
    e = cudaMemcpyFromSymbol(&h, g_noalloc_err, sizeof(int));
    if (e != cudaSuccess) return ic::cuda_fail(nullptr, e, "noalloc status: read error word");
    if (h == 0) return IC_OK;
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_noalloc_err, &zero, sizeof(int));
    if (e != cudaSuccess) return ic::cuda_fail(nullptr, e, "noalloc status: clear error word");
    return ic::device_error(nullptr, h);
}
