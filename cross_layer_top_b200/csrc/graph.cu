// Stack graphs: one F/S layer stack ("IndexCache: Accelerating Sparse
// Attention via Cross-Layer Index Reuse", Figure 2) captured once as a CUDA
// graph and replayed, so a decode step of many small dependent kernels pays
// one graph launch instead of one launch (and one host round of argument
// checks and tensor-map encodes) per kernel.
//
// ic_stack_graph_create runs the stack once eagerly on a context-owned
// stream (sizing every scratch buffer and setting every kernel attribute),
// then captures the same calls and instantiates the graph.  The graph holds
// the device pointers of that moment: the caller keeps the layer tensors,
// idx_cache and dims->seq_len alive and changes their contents, not their
// addresses, between replays.  While any graph exists, the context refuses
// to regrow the scratch buffers the graph uses.
//
// ic_stack_graph_create_ahead captures ic_run_stack_ahead instead: the side
// stream joins the capture through the fork event and rejoins it through
// the last F layer's event, so the graph holds both streams' kernels with
// the same dependencies.
#include "ic_internal.h"

using namespace ic;

struct ic_graph {
    ic_ctx* ctx = nullptr;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    int64_t kernels = 0;  // kernel launches in one replay
};

namespace {

// the stack in the chosen schedule: ic_run_stack, or ic_run_stack_ahead
// when idx_cache2 is given
int run_schedule(ic_ctx* ctx, const ic_pattern* pattern, const ic_layer_io* layers,
                 const ic_stack_dims* dims, int32_t* idx_cache, int32_t* idx_cache2,
                 cudaStream_t s) {
    if (idx_cache2) return ic_run_stack_ahead(ctx, pattern, layers, dims, idx_cache, idx_cache2, s);
    return ic_run_stack(ctx, pattern, layers, dims, idx_cache, s);
}

int graph_create(ic_ctx* ctx, const ic_pattern* pattern, const ic_layer_io* layers,
                 const ic_stack_dims* dims, int32_t* idx_cache, int32_t* idx_cache2,
                 ic_graph** out) {
    if (!out) return fail(ctx, IC_ERR_INVALID_ARG, "stack_graph_create: out is NULL");
    *out = nullptr;
    int rc = check_stack_args(ctx, pattern, layers, dims, idx_cache);
    if (rc) return rc;
    cudaSetDevice(ctx->device);
    cudaStream_t s = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "stack_graph_create: stream");
    const bool timing = ctx->timing;
    ctx->timing = false;  // no timing events inside the graph
    // eager pass: scratch sizes, kernel attributes, cluster-occupancy queries
    rc = run_schedule(ctx, pattern, layers, dims, idx_cache, idx_cache2, s);
    if (!rc) {
        e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) rc = cuda_fail(ctx, e, "stack_graph_create: eager pass");
    }
    ic_graph* g = nullptr;
    if (!rc) {
        g = new ic_graph();
        g->ctx = ctx;
        const int64_t before = ctx->launch_count;
        e = cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal);
        if (e != cudaSuccess) {
            rc = cuda_fail(ctx, e, "stack_graph_create: begin capture");
        } else {
            rc = run_schedule(ctx, pattern, layers, dims, idx_cache, idx_cache2, s);
            cudaGraph_t graph = nullptr;
            e = cudaStreamEndCapture(s, &graph);  // always ends the capture
            g->graph = graph;
            if (!rc && e != cudaSuccess) rc = cuda_fail(ctx, e, "stack_graph_create: end capture");
            if (!rc) {
                e = cudaGraphInstantiate(&g->exec, g->graph, 0);
                if (e != cudaSuccess) rc = cuda_fail(ctx, e, "stack_graph_create: instantiate");
            }
        }
        g->kernels = ctx->launch_count - before;
        ctx->launch_count = before;  // counted at replay instead
    }
    ctx->timing = timing;
    cudaStreamDestroy(s);
    if (rc) {
        if (g) {
            if (g->exec) cudaGraphExecDestroy(g->exec);
            if (g->graph) cudaGraphDestroy(g->graph);
            delete g;
        }
        cudaGetLastError();
        return rc;
    }
    ctx->graphs_alive++;
    *out = g;
    return IC_OK;
}

}  // namespace

extern "C" int ic_stack_graph_create(ic_ctx* ctx, const ic_pattern* pattern,
                                     const ic_layer_io* layers, const ic_stack_dims* dims,
                                     int32_t* idx_cache, ic_graph** out) {
    return graph_create(ctx, pattern, layers, dims, idx_cache, nullptr, out);
}

extern "C" int ic_stack_graph_create_ahead(ic_ctx* ctx, const ic_pattern* pattern,
                                           const ic_layer_io* layers, const ic_stack_dims* dims,
                                           int32_t* idx_cache, int32_t* idx_cache2,
                                           ic_graph** out) {
    if (!idx_cache2 || idx_cache2 == idx_cache)
        return fail(ctx, IC_ERR_INVALID_ARG, "stack_graph_create_ahead: idx_cache2 must be a "
                                             "second buffer");
    return graph_create(ctx, pattern, layers, dims, idx_cache, idx_cache2, out);
}

extern "C" int ic_stack_graph_launch(ic_graph* g, void* stream) {
    if (!g || !g->exec) return fail(nullptr, IC_ERR_INVALID_ARG, "stack_graph_launch: no graph");
    cudaSetDevice(g->ctx->device);
    cudaError_t e = cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(g->ctx, e, "stack_graph_launch");
    g->ctx->launch_count += g->kernels;
    return IC_OK;
}

extern "C" int64_t ic_stack_graph_kernels(const ic_graph* g) { return g ? g->kernels : -1; }

extern "C" int ic_stack_graph_destroy(ic_graph* g) {
    if (!g) return IC_ERR_INVALID_ARG;
    cudaSetDevice(g->ctx->device);
    if (g->exec) cudaGraphExecDestroy(g->exec);
    if (g->graph) cudaGraphDestroy(g->graph);
    g->ctx->graphs_alive--;
    delete g;
    return IC_OK;
}
