// ic_run_stack_ahead: the F/S layer stack ("IndexCache: Accelerating
// Sparse Attention via Cross-Layer Index Reuse", Figure 2) with each F
// layer's indexer and top-k issued ahead, on a second stream, while the
// attention of the layers before it runs: the scheduling of the multi-layer
// indexer page ("MLI"), without its change of what the indexer reads.  It
// is only a different order of the same kernels on the same inputs, valid
// because every F layer's indexer inputs are given to the stack rather than
// computed by the layers before it.
//
// Index tensors alternate between two buffers: the j-th F layer writes
// buf[j % 2] = (idx_cache, idx_cache2)[j % 2], and it and the S layers after
// it attend from there.  Streams:
//   side stream (context-owned): F layer j's indexer waits until buf[j % 2]
//     is free (the attention of every layer that read F layer j-2's indices
//     has run), writes it, and records indexed[j % 2];
//   caller's stream: each layer's attention waits indexed[j % 2] of its F
//     layer; after the last layer of F layer j's group it records freed[j % 2].
// So F layer j's indexer can run during the attention of F layer j-1's
// group.  The side stream first waits for everything the caller's stream
// held at the call, and the caller's stream ends after the last attention,
// which waited for the last indexer: completion of `stream` covers all work.
#include "ic_internal.h"

using namespace ic;

namespace {

int init_ahead(ic_ctx* ctx) {
    auto& a = ctx->ahead;
    if (a.ready) return IC_OK;
    cudaError_t e = cudaStreamCreateWithFlags(&a.side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a.start, cudaEventDisableTiming);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&a.indexed[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a.freed[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_ahead: stream / events");
    a.ready = true;
    return IC_OK;
}

}  // namespace

extern "C" int ic_run_stack_ahead(ic_ctx* ctx, const ic_pattern* pattern, const ic_layer_io* layers,
                                  const ic_stack_dims* dims, int32_t* idx_cache,
                                  int32_t* idx_cache2, void* stream) {
    int rc = check_stack_args(ctx, pattern, layers, dims, idx_cache);
    if (rc) return rc;
    if (!idx_cache2 || idx_cache2 == idx_cache)
        return fail(ctx, IC_ERR_INVALID_ARG, "run_stack_ahead: idx_cache2 must be a second buffer");
    cudaSetDevice(ctx->device);
    rc = init_ahead(ctx);
    if (rc) return rc;
    auto& a = ctx->ahead;
    const bool prefill = dims->mode == IC_PREFILL;
    const int rows = prefill ? dims->L : dims->B;
    const int k = dims->k;
    cudaStream_t main = reinterpret_cast<cudaStream_t>(stream);
    int32_t* buf[2] = {idx_cache, idx_cache2};
    // no programmatic launches or cross-layer prefetch: the kernels' order
    // across the two streams is set by the events alone
    ctx->pdl = 0;
    ctx->pf_K = ctx->pf_V = nullptr;
    cudaError_t e = cudaEventRecord(a.start, main);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(a.side, a.start, 0);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_ahead: fork");
    // On an error below, the caller's stream still waits for what the side
    // stream holds, so that nothing writes the caller's buffers after the
    // caller's stream has passed this call.
    struct Join {
        ic_ctx::Ahead& a;
        cudaStream_t main;
        bool armed = true;
        ~Join() {
            if (armed && cudaEventRecord(a.start, a.side) == cudaSuccess)
                cudaStreamWaitEvent(main, a.start, 0);
        }
    } join{a, main};
    const int N = static_cast<int>(pattern->c.size());
    int j = -1;  // F layers seen
    for (int l = 0; l < N; ++l) {
        const ic_layer_io& io = layers[l];
        if (pattern->c[l] == 'F') {
            ++j;
            const int b = j % 2;
            // F layer j-1's group has all its attention enqueued: its buffer
            // is free once that has run
            if (j >= 1) {
                e = cudaEventRecord(a.freed[(j - 1) % 2], main);
                if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_ahead: record freed");
            }
            if (j >= 2) {
                e = cudaStreamWaitEvent(a.side, a.freed[b], 0);
                if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_ahead: wait freed");
            }
            if (prefill)
                rc = ic_index_fp(ctx, io.qI, io.kI, io.w, dims->L, dims->H_I, dims->d_I, k, buf[b],
                                 a.side);
            else
                rc = ic_index_fp_decode(ctx, io.qI, io.w, io.kI8, io.kI_scale, dims->seq_len,
                                        dims->B, dims->S_max, dims->H_I, dims->d_I, k, buf[b],
                                        a.side);
            if (rc) return rc;
            e = cudaEventRecord(a.indexed[b], a.side);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(main, a.indexed[b], 0);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_ahead: indexed");
        }
        const int32_t* idx = nullptr;
        ic_index_reuse(buf[j % 2], &idx);
        if (io.idx_snapshot) {
            e = cudaMemcpyAsync(io.idx_snapshot, idx, static_cast<size_t>(rows) * k * sizeof(int32_t),
                                cudaMemcpyDeviceToDevice, main);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_ahead: snapshot copy");
        }
        if (prefill)
            rc = ic_sparse_attn(ctx, io.Q, io.K, io.V, idx, rows, dims->Hq, dims->d, k, 0, 0,
                                dims->L, dims->scale, io.out, main);
        else
            rc = ic_sparse_attn(ctx, io.Q, io.K, io.V, idx, rows, dims->Hq, dims->d, k, 1,
                                static_cast<int64_t>(dims->S_max) * dims->d, dims->S_max,
                                dims->scale, io.out, main);
        if (rc) return rc;
    }
    join.armed = false;  // the last layer waited for the last indexer
    return IC_OK;
}
