// ic_run_stack_host: the F/S layer stack ("IndexCache: Accelerating Sparse
// Attention via Cross-Layer Index Reuse", Figure 2) on inputs that live in
// host memory, with the host<->device copies overlapped with the compute.
//
// The context stages the layers through n = 4 device slots.  Layer l uses
// slot l % n:
//   copy-in stream : wait until layer l-n has computed (its inputs are no
//                    longer read), copy layer l's inputs in, record in_ready;
//   caller's stream: wait in_ready and until layer l-n's output has been
//                    copied out, run the layer, record computed;
//   copy-out stream: wait computed, copy the output to host, record out_done.
// So later layers' inputs cross PCIe while layer l computes, and layer l's
// output crosses back while the next layers compute.  With two slots the
// copy-in stream would idle behind every layer that computes longer than
// the next layer's inputs take to copy (an F layer followed by S layers).  The events persist in the
// context, which also orders consecutive calls.  At the end the caller's
// stream waits for the last outputs, so its completion means every output
// is in host memory.
#include "ic_internal.h"

using namespace ic;

namespace {

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Byte sizes of one layer's fields, from the stack dimensions.
struct FieldSizes {
    size_t qI, kI, w, kI8, kI_scale, Q, K, V, out;
    size_t total() const {
        return align256(qI) + align256(kI) + align256(w) + align256(kI8) + align256(kI_scale) +
               align256(Q) + align256(K) + align256(V) + align256(out);
    }
};

FieldSizes field_sizes(const ic_stack_dims* d) {
    FieldSizes f{};
    const size_t bf = 2;
    if (d->mode == IC_PREFILL) {
        const size_t L = static_cast<size_t>(d->L);
        f.qI = L * d->H_I * d->d_I * bf;
        f.kI = L * d->d_I * bf;
        f.w = L * d->H_I * bf;
        f.Q = L * d->Hq * d->d * bf;
        f.K = f.V = L * d->d * bf;
        f.out = L * d->Hq * d->d * bf;
    } else {
        const size_t B = static_cast<size_t>(d->B), S = static_cast<size_t>(d->S_max);
        f.qI = B * d->H_I * d->d_I * bf;
        f.w = B * d->H_I * bf;
        f.kI8 = B * S * d->d_I;
        f.kI_scale = B * S * 4;
        f.Q = B * d->Hq * d->d * bf;
        f.K = f.V = B * S * d->d * bf;
        f.out = B * d->Hq * d->d * bf;
    }
    return f;
}

int init_host_stack(ic_ctx* ctx) {
    auto& hs = ctx->hs;
    if (hs.ready) return IC_OK;
    cudaError_t e = cudaStreamCreateWithFlags(&hs.in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hs.out, cudaStreamNonBlocking);
    for (int i = 0; i < ic_ctx::kHostSlots && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&hs.in_ready[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hs.computed[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hs.out_done[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_host: streams / events");
    hs.ready = true;
    return IC_OK;
}

}  // namespace

extern "C" int ic_run_stack_host(ic_ctx* ctx, const ic_pattern* pattern,
                                 const ic_layer_io* layers_host, const ic_stack_dims* dims,
                                 int32_t* idx_cache, void* stream) {
    int rc = check_stack_args(ctx, pattern, layers_host, dims, idx_cache);
    if (rc) return rc;
    cudaSetDevice(ctx->device);
    rc = init_host_stack(ctx);
    if (rc) return rc;
    auto& hs = ctx->hs;
    const FieldSizes fs = field_sizes(dims);
    const size_t need = fs.total();
    if (need > hs.slot_cap) {
        // the slots are about to be replaced: nothing may still use the old ones
        cudaError_t e = cudaStreamSynchronize(hs.in);
        if (e == cudaSuccess) e = cudaStreamSynchronize(hs.out);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_host: drain before regrow");
        for (int i = 0; i < ic_ctx::kHostSlots; ++i) {
            cudaFree(hs.slot[i]);
            hs.slot[i] = nullptr;
        }
        hs.slot_cap = 0;
        for (int i = 0; i < ic_ctx::kHostSlots; ++i) {
            e = cudaMalloc(&hs.slot[i], need);
            if (e != cudaSuccess) {
                for (int j = 0; j < ic_ctx::kHostSlots; ++j) {
                    cudaFree(hs.slot[j]);
                    hs.slot[j] = nullptr;
                }
                cudaGetLastError();
                return fail(ctx, IC_ERR_NOMEM, "run_stack_host: %d slots of %zu bytes",
                            ic_ctx::kHostSlots, need);
            }
        }
        hs.slot_cap = need;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // On an error below, `stream` still waits for every copy already issued
    // on the context's streams, so that none reads or writes the caller's
    // host buffers after the caller's stream has passed this call.
    struct Join {
        ic_ctx::HostStack& hs;
        cudaStream_t s;
        bool armed = true;
        ~Join() {
            if (!armed) return;
            if (cudaEventRecord(hs.in_ready[0], hs.in) == cudaSuccess)
                cudaStreamWaitEvent(s, hs.in_ready[0], 0);
            if (cudaEventRecord(hs.out_done[0], hs.out) == cudaSuccess)
                cudaStreamWaitEvent(s, hs.out_done[0], 0);
        }
    } join{hs, s};
    const int N = static_cast<int>(pattern->c.size());
    for (int l = 0; l < N; ++l) {
        const int sl = l % ic_ctx::kHostSlots;
        const ic_layer_io& h = layers_host[l];
        if (!h.Q || !h.K || !h.V || !h.out)
            return fail(ctx, IC_ERR_INVALID_ARG, "run_stack_host: layer %d lacks Q/K/V/out", l);
        // this layer's device view of the slot
        char* p = static_cast<char*>(hs.slot[sl]);
        ic_layer_io d{};
        auto take = [&](size_t bytes) {
            void* q = p;
            p += align256(bytes);
            return q;
        };
        void* dqI = take(fs.qI);
        void* dkI = take(fs.kI);
        void* dw = take(fs.w);
        void* dkI8 = take(fs.kI8);
        void* dks = take(fs.kI_scale);
        void* dQ = take(fs.Q);
        void* dK = take(fs.K);
        void* dV = take(fs.V);
        void* dout = take(fs.out);
        cudaError_t e = cudaStreamWaitEvent(hs.in, hs.computed[sl], 0);
        struct Copy {
            const void* src;
            void* dst;
            size_t bytes;
        };
        const Copy copies[] = {{h.qI, dqI, fs.qI},     {h.kI, dkI, fs.kI},
                               {h.w, dw, fs.w},        {h.kI8, dkI8, fs.kI8},
                               {h.kI_scale, dks, fs.kI_scale}, {h.Q, dQ, fs.Q},
                               {h.K, dK, fs.K},        {h.V, dV, fs.V}};
        for (const Copy& c : copies)
            if (e == cudaSuccess && c.src && c.bytes)
                e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess) e = cudaEventRecord(hs.in_ready[sl], hs.in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hs.in_ready[sl], 0);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hs.out_done[sl], 0);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_host: copy in");
        d.qI = h.qI ? dqI : nullptr;
        d.kI = h.kI ? dkI : nullptr;
        d.w = h.w ? dw : nullptr;
        d.kI8 = h.kI8 ? static_cast<const uint8_t*>(dkI8) : nullptr;
        d.kI_scale = h.kI_scale ? static_cast<const float*>(dks) : nullptr;
        d.Q = dQ;
        d.K = dK;
        d.V = dV;
        d.out = dout;
        d.idx_snapshot = h.idx_snapshot;  // device memory, as in ic_run_stack
        rc = run_stack_layer(ctx, pattern->c[l], d, nullptr, dims, idx_cache, stream);
        if (rc) return rc;
        e = cudaEventRecord(hs.computed[sl], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.out, hs.computed[sl], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(h.out, dout, fs.out, cudaMemcpyDeviceToHost, hs.out);
        if (e == cudaSuccess) e = cudaEventRecord(hs.out_done[sl], hs.out);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_host: copy out");
    }
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < ic_ctx::kHostSlots && e == cudaSuccess; ++i)
        e = cudaStreamWaitEvent(s, hs.out_done[i], 0);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "run_stack_host: final wait");
    join.armed = false;  // the caller's stream has waited for every copy already
    return IC_OK;
}
