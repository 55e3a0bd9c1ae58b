/*
 * indexcache.h — C ABI of libindexcache.so, the B200 (sm_100a) hot path of
 * DeepSeek Sparse Attention with IndexCache (cross-layer top-k index reuse).
 *
 * The operations follow two web pages, cited by title and section:
 *   [IC] "IndexCache: Accelerating Sparse Attention via Cross-Layer Index
 *        Reuse" (paper summary): method details (pattern c in {F,S}^N,
 *        f(l) = max{j<l : c_j = F}, first layer F), Figure 2 (inference
 *        loop: F layers run the indexer and top-k and overwrite the cache,
 *        S layers copy the cached indices, every layer runs sparse
 *        attention), §2.1 (top-k with k = 2048, FP8 indexer arithmetic),
 *        §3.1.1 (uniform interleave).
 *   [RN] "IndexCache：跨层复用稀疏索引，以及它为什么能被训练" (reading notes):
 *        §2.1 indexer score I[t,s] = sum_j w[t,j] ReLU(q_I[t,j] . k_I[s]);
 *        §2.2 the cache holds the current index tensor only; §3 sparse
 *        attention o_t = sum_{s in T_t} softmax(Q_t.K_s/sqrt(d)) V_s;
 *        §10.1 decode scans the whole indexer key cache per token; §11 S
 *        layers keep no indexer key cache.
 *
 * Conventions (all calls):
 *  - Tensors are caller-owned DEVICE pointers, row-major and contiguous,
 *    with the sizes passed explicitly.  bf16 tensors are passed as void*.
 *    Tensors read by TMA (q_I, k_I) must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  They return after enqueueing work.
 *  - Every call returns IC_OK (0) or an IC_ERR_* code and never throws.  The
 *    message of the last failure is ic_last_error(ctx).  Argument errors are
 *    detected on the host before anything is enqueued.  Errors found on the
 *    device (a bounded wait that ran out, an index outside [-1, kv_len))
 *    are latched in the context and reported by ic_sync_status().
 *  - Positions are 0-based; causal means s <= t (the query sees itself).
 *  - Index rows hold min(k, n) selected positions in ascending order
 *    followed by -1 padding; ties in score go to the lower position.
 *  - A context (ic_ctx) owns scratch memory (fp32 score rows; the staging
 *    slots of ic_run_stack_host), timing events and the device error flag.
 *    It is not thread-safe: use one context per host thread / stream.
 */
#ifndef INDEXCACHE_H
#define INDEXCACHE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define IC_OK 0
#define IC_ERR_INVALID_ARG 1  /* null pointer, negative size, misaligned pointer */
#define IC_ERR_PATTERN 2      /* pattern not over {F,S} or first layer not F */
#define IC_ERR_SHAPE 3        /* inconsistent sizes (e.g. k < 1) */
#define IC_ERR_UNSUPPORTED 4  /* a size outside what the kernels are built for */
#define IC_ERR_CUDA 5         /* a CUDA runtime/driver call failed */
#define IC_ERR_TIMEOUT 6      /* a bounded device wait ran out */
#define IC_ERR_NOMEM 7        /* scratch allocation failed */
#define IC_ERR_DEVICE 8       /* a device-side check failed (bad index) */

#define IC_PREFILL 0
#define IC_DECODE 1

/* Kernel ids for the timing counters. */
#define IC_K_INDEX_SCORE 0        /* prefill indexer score (tcgen05) */
#define IC_K_INDEX_SCORE_DECODE 1 /* decode FP8 indexer-key scan (tcgen05) */
#define IC_K_TOPK 2               /* per-row top-k select */
#define IC_K_ATTN 3               /* sparse MQA attention (gather + softmax) */
#define IC_K_OVERLAP 4            /* cross-layer index overlap (diagnostic) */
#define IC_K_COUNT 5

typedef struct ic_ctx ic_ctx;
typedef struct ic_pattern ic_pattern;

/* ---------------------------------------------------------------- context */

/* Library version, major*10000 + minor*100 + patch. */
int ic_version(void);

/* Create a context on CUDA `device`.  `scratch_bytes` bounds the score
 * scratch used by ic_index_fp (0 = 2 GiB); rows are processed in chunks
 * that fit.  Scratch is allocated lazily on first use.  *out receives the
 * context.  Errors: IC_ERR_INVALID_ARG (out NULL), IC_ERR_CUDA. */
int ic_ctx_create(ic_ctx **out, int device, size_t scratch_bytes);

/* Free the context and its scratch (synchronizes the device first). */
int ic_ctx_destroy(ic_ctx *ctx);

/* Message of the last failure on `ctx` (or of the last ic_ctx_create /
 * ic_create_pattern failure when ctx is NULL).  Never NULL. */
const char *ic_last_error(const ic_ctx *ctx);

/* Synchronize `stream`, then read and clear the context's device error
 * flag.  Returns IC_OK, IC_ERR_TIMEOUT, IC_ERR_DEVICE or IC_ERR_CUDA. */
int ic_sync_status(ic_ctx *ctx, void *stream);

/* Kernel timing counters (tracing).  When enabled, every kernel the context
 * launches is bracketed by CUDA events on its launch stream.
 * ic_ctx_get_timing synchronizes on the last recorded event and returns the
 * summed device time (ms) and launch count for kernel id `kernel`.
 * ic_ctx_reset_timing clears all counters. */
int ic_ctx_set_timing(ic_ctx *ctx, int enable);
int ic_ctx_get_timing(ic_ctx *ctx, int kernel, double *total_ms, int64_t *launches);
int ic_ctx_reset_timing(ic_ctx *ctx);
/* Number of kernels this context has launched since creation (all ids). */
int64_t ic_ctx_launch_count(const ic_ctx *ctx);

/* ---------------------------------------------------------------- pattern */

/* [IC] method details: parse c[0..n_layers) over {'F','S'}; c[0] must be
 * 'F'.  Errors: IC_ERR_INVALID_ARG, IC_ERR_PATTERN.  Host only. */
int ic_create_pattern(const char *c, int n_layers, ic_pattern **out);

/* [IC] §3.1.1 uniform interleave: layer l is F iff l % r == 0. */
int ic_pattern_uniform(int n_layers, int r, ic_pattern **out);

int ic_pattern_destroy(ic_pattern *p);
int ic_pattern_size(const ic_pattern *p);                     /* n_layers, or -1 */
int ic_pattern_string(const ic_pattern *p, char *buf, int buflen); /* NUL-terminated */

/* src_out[l] = l for an F layer, f(l) = max{j<l : c_j=F} for an S layer.
 * src_out is a HOST array of n_layers ints. */
int ic_pattern_src(const ic_pattern *p, int32_t *src_out);

/* ------------------------------------------------------- prefill indexer */

/* [RN] §2.1 lightning-indexer scores of query rows t in [row_begin,row_end):
 *   scores[(t - row_begin)*ld + s] = sum_j w[t,j] * ReLU(q_I[t,j,:] . k_I[s,:])
 * for s <= t; entries with s > t are not written.
 *   q_I: bf16 [L, H_I, d_I];  k_I: bf16 [L, d_I];  w: bf16 [L, H_I].
 *   scores: fp32, ld >= row_end, ld % 4 == 0.
 * Supported: H_I in {4,8,16,32,64}, d_I in {32,64,128}.  fp32 accumulation
 * on the tensor cores; exact whenever every partial sum is (e.g. small
 * integers).  Errors: IC_ERR_INVALID_ARG, IC_ERR_UNSUPPORTED, IC_ERR_CUDA. */
int ic_index_score(ic_ctx *ctx, const void *qI, const void *kI, const void *w, int L, int H_I,
                   int d_I, int row_begin, int row_end, float *scores, int64_t ld, void *stream);

/* Per-row top-k ([IC] notation T_t = Top-k(I_t)).  Row r has n_r candidates
 * scores[r*ld + 0 .. n_r-1], with n_r = row_len[r] when row_len (device,
 * int32 [rows]) is non-NULL, else n_r = causal_base + r + 1.  Writes
 * idx_out[r*ld_out + 0..k-1]: the min(k, n_r) positions of the largest
 * scores, ascending, ties to the lower position, then -1.  Rows with
 * n_r <= k read no scores.  1 <= k <= 2048.  -0.0 equals +0.0. */
int ic_topk(ic_ctx *ctx, const float *scores, int64_t ld, int rows, int k, int causal_base,
            const int32_t *row_len, int32_t *idx_out, int64_t ld_out, void *stream);

/* One prefill F layer ([IC] Figure 2, steps "I <- INDEXER(X); T <-
 * Top-k(I); cache <- T"): idx_out int32 [L, k] (the index cache) receives
 * T_t for every t.  Rows t < k need no score (T_t = {0..t}).  Scores go
 * through the context's scratch in row chunks. */
int ic_index_fp(ic_ctx *ctx, const void *qI, const void *kI, const void *w, int L, int H_I,
                int d_I, int k, int32_t *idx_out, void *stream);

/* FP8 prefill indexer ([IC] §2.1: the lightning indexer runs in FP8).  The
 * same score as ic_index_score on dequantised inputs:
 *   I[t,s] = sum_j w[t,j] * ReLU((e4m3(qI8[t,j,:]) q_scale[t,j])
 *                                 . (e4m3(kI8[s,:]) k_scale[s]))
 *          = k_scale[s] * sum_j (w[t,j] q_scale[t,j]) * ReLU(e4m3(qI8[t,j,:]) . e4m3(kI8[s,:]))
 * (the scales must be > 0, which makes the two forms equal).  The products of
 * e4m3 values are exact and accumulate in fp32 on the tensor cores
 * (kind::f8f6f4).
 *   qI8: e4m3 bytes [L, H_I, d_I]; q_scale: fp32 [L, H_I] (> 0);
 *   kI8: e4m3 bytes [L, d_I];      k_scale: fp32 [L] (> 0);  w: bf16 [L, H_I].
 *   scores: fp32, ld >= row_end, ld % 4 == 0.
 * Supported: H_I in {16,32,64}, d_I = 128.  Errors as ic_index_score. */
int ic_index_score_fp8(ic_ctx *ctx, const uint8_t *qI8, const float *q_scale, const uint8_t *kI8,
                       const float *k_scale, const void *w, int L, int H_I, int d_I, int row_begin,
                       int row_end, float *scores, int64_t ld, void *stream);

/* FP8 prefill F layer: ic_index_fp on the scores of ic_index_score_fp8. */
int ic_index_fp_fp8(ic_ctx *ctx, const uint8_t *qI8, const float *q_scale, const uint8_t *kI8,
                    const float *k_scale, const void *w, int L, int H_I, int d_I, int k,
                    int32_t *idx_out, void *stream);

/* S layer ([IC] Figure 2 "T <- cache"): the cached tensor itself is used, no
 * copy and no kernel.  *idx_out = idx_cache. */
int ic_index_reuse(const int32_t *idx_cache, const int32_t **idx_out);

/* -------------------------------------------------------- decode indexer */

/* [RN] §2.1 score for one new query per sequence against its FP8 indexer
 * key cache ([IC] §2.1 FP8 indexer; [RN] §10.1 full scan per token):
 *   scores[b*ld + s] = sum_j w[b,j] * ReLU(q[b,j,:] . (e4m3(kI8[b,s,:]) * kI_scale[b,s]))
 * for s < seq_len[b].  q: bf16 [B, H_I, d_I]; w: bf16 [B, H_I];
 * kI8: e4m3 bytes [B, S_max, d_I]; kI_scale: fp32 [B, S_max], > 0;
 * seq_len: device int32 [B], 1 <= seq_len[b] <= S_max.  ld >= S_max.
 * Supported: H_I in {32,64}, d_I = 128. */
int ic_index_score_decode(ic_ctx *ctx, const void *q, const void *w, const uint8_t *kI8,
                          const float *kI_scale, const int32_t *seq_len, int B, int S_max, int H_I,
                          int d_I, float *scores, int64_t ld, void *stream);

/* Decode F layer: scores then top-k over each sequence's seq_len[b]
 * candidates; idx_out int32 [B, k]. */
int ic_index_fp_decode(ic_ctx *ctx, const void *q, const void *w, const uint8_t *kI8,
                       const float *kI_scale, const int32_t *seq_len, int B, int S_max, int H_I,
                       int d_I, int k, int32_t *idx_out, void *stream);

/* Allocation-free variant of ic_index_fp_decode, for callers that cannot
 * call cudaMalloc on their decode path: engines that give all free HBM to
 * their own KV-cache pool (an allocation could fail, and it synchronizes the
 * device in a latency-bound per-token loop), or a decode step replayed from
 * a captured stream.  The pages have no counterpart to this entry point.
 * Same arguments, results and support as ic_index_fp_decode, without a
 * context.  The fp32 score rows live in a fixed 16 MiB array in the
 * library's device memory (every GPU that loads the library holds it until
 * exit): B * round_up(S_max, 64) must be <= 4194304, else IC_ERR_UNSUPPORTED
 * with a message.  The first call on a device resolves that array's address
 * (cudaGetSymbolAddress) and should come before any stream capture.  All
 * calls share the array: calls whose kernels overlap on the GPU race.  The
 * host side of a call holds a per-device lock, so host threads may call it
 * concurrently.  The call never synchronizes: errors found on the device (a
 * bounded wait that ran out, a misaligned shared-memory window) are latched
 * in a device word of the library, which ic_noalloc_sync_status reports;
 * after such an error the indices of the calls before that report are not
 * valid.  Error messages: ic_last_error(NULL). */
int ic_index_fp_decode_noalloc(const void *q, const void *w, const uint8_t *kI8,
                               const float *kI_scale, const int32_t *seq_len, int B, int S_max,
                               int H_I, int d_I, int k, int32_t *idx_out, void *stream);

/* Status of ic_index_fp_decode_noalloc on the current device, also without
 * allocating: synchronizes `stream`, then reads and clears the device error
 * word that the allocation-free path's kernels latch (copies between a host
 * int and the library's device symbol).  Returns IC_OK, IC_ERR_TIMEOUT,
 * IC_ERR_DEVICE or IC_ERR_CUDA; message in ic_last_error(NULL).  Like the
 * entry point it reports on, it has no counterpart on the pages. */
int ic_noalloc_sync_status(void *stream);

/* ------------------------------------------ prefill split across ranks */

/* The prefill path splits by query rows: given the whole k_I, K and V, every
 * row's scores, top-k and attention need nothing from any other row ([RN]
 * §2.1 and §3: each query row's score row and softmax are its own; [RN]
 * §10.3 reports the pages' prefill with data-parallel attention over 8
 * GPUs).  A rank owns some row ranges; one all-gather of its rows of k_I, K
 * and V (done by the caller, e.g. torch.distributed over NCCL) gives every
 * rank the whole key tensors, and from there everything is local. */

/* Causal-balanced split of L query rows over `world` ranks.  The rows are cut
 * into 2*world chunks of near-equal size (the first L % (2*world) chunks one
 * row longer); rank `rank` owns chunks rank and 2*world-1-rank, so each rank
 * pairs an early, cheap chunk with a late, costly one (an F-layer row t
 * scores t+1 keys).  Writes ranges[0..3] = {a0, b0, a1, b1} (half-open row
 * ranges, b0 <= a1; a range is empty when L < 2*world) and *n_ranges = 2.
 * Host only.
 * Errors: IC_ERR_INVALID_ARG (NULL, L < 0, world < 1, rank outside). */
int ic_prefill_partition(int L, int world, int rank, int32_t *ranges, int *n_ranges);

/* One prefill F layer for the query rows [row_begin, row_end) only, with
 * their q_I and w rows held compactly:
 *   qI_rows: bf16 [row_end - row_begin, H_I, d_I];  w_rows: bf16 [.., H_I];
 *   kI: bf16 [L, d_I], the whole key tensor (rows >= row_end are not read);
 *   idx_out: int32 [row_end - row_begin, k]: row i holds T_{row_begin + i}.
 * Results are identical to the same rows of ic_index_fp.  An empty range
 * returns IC_OK at once.  Supported and errors as ic_index_fp, plus
 * IC_ERR_SHAPE for a range outside [0, L). */
int ic_index_fp_rows(ic_ctx *ctx, const void *qI_rows, const void *w_rows, const void *kI, int L,
                     int H_I, int d_I, int row_begin, int row_end, int k, int32_t *idx_out,
                     void *stream);

/* ------------------------------------------------------ sparse attention */

/* [RN] §3 sparse MQA attention, every layer:
 *   out[r,h,:] = sum_{s in idx[r,:], s >= 0} softmax_s(scale * Q[r,h,:].K[s,:]) V[s,:]
 * Q: bf16 [rows, Hq, d]; out: bf16 [rows, Hq, d]; idx: int32 [rows, k].
 * K, V: bf16; query row r reads the block of sequence r / rows_per_seq at
 * K + (r / rows_per_seq) * kv_seq_stride (elements), whose rows are
 * [kv_len, d].  One shared K/V head.  Entries -1 are skipped; an entry
 * outside [-1, kv_len) is skipped and latched as IC_ERR_DEVICE.  A row with
 * no valid entry produces zeros.  scale <= 0 means 1/sqrt(d).
 * Supported: d in {64,128}, 1 <= Hq <= 16, 1 <= k <= 2048.  Q, K, V 16-byte
 * aligned, out 8-byte aligned (else IC_ERR_INVALID_ARG). */
int ic_sparse_attn(ic_ctx *ctx, const void *Q, const void *K, const void *V, const int32_t *idx,
                   int rows, int Hq, int d, int k, int rows_per_seq, int64_t kv_seq_stride,
                   int kv_len, float scale, void *out, void *stream);

/* ------------------------------------------------ cross-layer overlap */

/* [IC] Appendix A, [RN] §3.2: how far two layers' top-k sets agree, the
 * quantity that makes reusing one layer's indices in the next workable.
 *   hits[r] = |{x : idx_a[r,x] >= 0 and idx_a[r,x] occurs in idx_b[r,:]}|
 * and the overlap of row r is hits[r] / k.  idx_a, idx_b: device int32
 * [rows, k], contiguous, entries in [0, n_keys) or -1 (never counted), in any
 * order; an entry of idx_a counts once per occurrence.  hits: device int32
 * [rows], written by this call.  An entry outside [-1, n_keys) is skipped and
 * latched as IC_ERR_DEVICE.  Supported: 1 <= n_keys <= 6553600, k >= 1. */
int ic_index_overlap(ic_ctx *ctx, const int32_t *idx_a, const int32_t *idx_b, int rows, int k,
                     int n_keys, int32_t *hits, void *stream);

/* ------------------------------------------------------------ layer stack */

typedef struct ic_layer_io {
    /* F layers only (NULL on S layers, [RN] §11: S layers own no indexer).
     * prefill: qI bf16 [L,H_I,d_I], kI bf16 [L,d_I], w bf16 [L,H_I].
     * decode:  qI bf16 [B,H_I,d_I] (the new token's query), w bf16 [B,H_I],
     *          kI8 e4m3 [B,S_max,d_I], kI_scale fp32 [B,S_max]. */
    const void *qI;
    const void *kI;
    const void *w;
    const uint8_t *kI8;
    const float *kI_scale;
    /* every layer: Q bf16 [rows,Hq,d]; K, V bf16 (prefill [L,d], decode
     * [B,S_max,d]); out bf16 [rows,Hq,d]. */
    const void *Q;
    const void *K;
    const void *V;
    void *out;
    /* optional: device int32 [rows,k] that receives a copy of the index
     * tensor this layer attended with (for checking the reuse invariant). */
    int32_t *idx_snapshot;
} ic_layer_io;

typedef struct ic_stack_dims {
    int mode;               /* IC_PREFILL or IC_DECODE */
    int L;                  /* prefill: sequence length (rows = L) */
    int B;                  /* decode: sequences (rows = B) */
    int S_max;              /* decode: capacity of each sequence's caches */
    const int32_t *seq_len; /* decode: device int32 [B], candidates incl. the new token */
    int H_I, d_I, k, Hq, d;
    float scale;            /* softmax scale; <= 0 means 1/sqrt(d) */
} ic_stack_dims;

/* [IC] Figure 2: for l = 0..N-1, if c_l = F run the indexer and top-k into
 * idx_cache (device int32 [rows, k], overwritten), else reuse idx_cache as
 * it stands; then sparse attention of layer l with its own Q/K/V at those
 * indices.  Everything is enqueued on `stream` with no host sync.
 * Decode stacks with B * 8 <= the SM count launch each kernel as a
 * programmatic dependent of the one before it: a kernel may start before
 * its predecessor in the stream finishes, but reads nothing a previous
 * kernel writes until that predecessor has completed, except that an S
 * layer's attention reads the index cache and prefetches (into L2 only) the
 * K/V rows at those slots first.  Larger decode batches launch normally;
 * there an attention layer followed by an S layer prefetches (into L2 only)
 * that layer's K/V rows at the shared slots after its own gather (a
 * prefetch changes no result).  A caller's own kernel before the stack is
 * always complete before the stack reads anything. */
int ic_run_stack(ic_ctx *ctx, const ic_pattern *pattern, const ic_layer_io *layers,
                 const ic_stack_dims *dims, int32_t *idx_cache, void *stream);

/* The same stack with every F layer's indexer and top-k issued ahead on a
 * second, context-owned stream, so that it runs while the attention of the
 * layers before it runs (the scheduling idea of the multi-layer indexer
 * page, "MLI", on this method's own indices).  Valid only because each F
 * layer's indexer inputs are given: in a model whose layer l reads layer
 * l-1's output this order would not exist.  The j-th F layer (0-based)
 * writes its index tensor to idx_cache when j is even and to idx_cache2
 * when j is odd (both device int32 [rows, k], distinct, overwritten), and
 * it and the S layers after it attend from there; F layer j's indexer
 * waits until the layers of F layer j-2's group have attended.  Every
 * output, snapshot and index tensor is bit-identical to ic_run_stack's.
 * The side stream first waits for the work `stream` held at the call, and
 * `stream` ends after the last layer, so its completion covers all work.
 * No programmatic launches or cross-layer prefetch.  Errors as ic_run_stack,
 * plus IC_ERR_INVALID_ARG when idx_cache2 is NULL or equals idx_cache; on an
 * error after work was issued, `stream` still waits for the side stream's
 * work, so completion of `stream` covers it. */
int ic_run_stack_ahead(ic_ctx *ctx, const ic_pattern *pattern, const ic_layer_io *layers,
                       const ic_stack_dims *dims, int32_t *idx_cache, int32_t *idx_cache2,
                       void *stream);

/* The prefill stack of one rank of a row split ([IC] Figure 2 over the
 * rank's rows).  `ranges` (HOST int32 [2*n_ranges], half-open, disjoint,
 * e.g. from ic_prefill_partition) are the rank's query rows.  In layers[l],
 * qI, w, Q, out and idx_snapshot hold the rank's rows only, range after
 * range in the order given (rows = the sum of the range lengths); kI, K and
 * V hold all dims->L rows (after the caller's all-gather).  idx_cache is
 * int32 [rows, k].  Every index row is identical to the same row of
 * ic_run_stack on the whole sequence, and so is every output row unless one
 * of the two attention launches is short enough (fewer rows than about
 * three CTAs per SM) to spread each row over a cluster of CTAs, which rounds
 * differently within the attention tolerance.  Prefill mode only. */
int ic_run_stack_rows(ic_ctx *ctx, const ic_pattern *pattern, const ic_layer_io *layers,
                      const ic_stack_dims *dims, const int32_t *ranges, int n_ranges,
                      int32_t *idx_cache, void *stream);

/* A stack captured once as a CUDA graph and replayed: a decode step of
 * many small dependent kernels then costs one graph launch.  Create runs
 * ic_run_stack once eagerly (sizing scratch, setting kernel attributes),
 * then captures the same calls; the graph keeps the device pointers of
 * layers, dims->seq_len and idx_cache as they are now, so the caller keeps
 * those buffers alive and changes only their contents between launches.
 * While a graph of ctx exists, calls that would need larger scratch than it
 * captured fail with IC_ERR_NOMEM.  Launch is asynchronous on `stream`.
 * ic_stack_graph_kernels: kernel launches in one replay.  Destroy before
 * ic_ctx_destroy. */
typedef struct ic_graph ic_graph;
int ic_stack_graph_create(ic_ctx *ctx, const ic_pattern *pattern, const ic_layer_io *layers,
                          const ic_stack_dims *dims, int32_t *idx_cache, ic_graph **out);
/* The same for the schedule of ic_run_stack_ahead (its two index buffers;
 * the side stream's kernels are captured into the same graph with their
 * dependencies).  Errors as ic_stack_graph_create, plus IC_ERR_INVALID_ARG
 * when idx_cache2 is NULL or equals idx_cache. */
int ic_stack_graph_create_ahead(ic_ctx *ctx, const ic_pattern *pattern, const ic_layer_io *layers,
                                const ic_stack_dims *dims, int32_t *idx_cache, int32_t *idx_cache2,
                                ic_graph **out);
int ic_stack_graph_launch(ic_graph *graph, void *stream);
int64_t ic_stack_graph_kernels(const ic_graph *graph);
int ic_stack_graph_destroy(ic_graph *graph);

/* The same stack on inputs in host memory, with the copies overlapped with
 * the compute.  Every pointer of layers_host[l] that ic_run_stack reads on
 * the device (qI, kI, w, kI8, kI_scale, Q, K, V) is read from host memory
 * instead, and out receives the layer's output in host memory; use pinned
 * (page-locked) host memory, or the copies neither overlap nor run at full
 * speed.  idx_snapshot (optional), idx_cache and dims->seq_len stay on the
 * device.  The context stages layers through four device slots, each sized
 * for the largest layer (allocated on first use, grown when dims grow):
 * later layers' inputs are copied in on a context-owned stream while layer l
 * computes on `stream` (layer l+4 waits for slot l % 4 to be free), and layer
 * l's output is copied out on another context-owned stream while the next
 * layers compute.  Asynchronous: when `stream` reaches the point after this
 * call, every output is in host memory; the host inputs must not change
 * before then.  Errors as ic_run_stack, plus IC_ERR_NOMEM when the four
 * slots cannot be allocated; on an error after copies were issued, `stream`
 * still waits for them, so its completion means no copy is left. */
int ic_run_stack_host(ic_ctx *ctx, const ic_pattern *pattern, const ic_layer_io *layers_host,
                      const ic_stack_dims *dims, int32_t *idx_cache, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* INDEXCACHE_H */
