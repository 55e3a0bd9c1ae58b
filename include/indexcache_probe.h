/*
 * indexcache_probe.h — libindexcache_probe.so, a separate measurement and
 * test library beside libindexcache.so (not part of the IndexCache method;
 * the pages have no counterpart).  It links against libindexcache.so, whose
 * contexts ic_probe_wait_timeout takes.
 *
 * ic_probe_gather enqueues a kernel that performs exactly the K/V row
 * gather of sparse attention and nothing else: for each of `rows` query
 * rows it copies the k rows K[idx[r, j]], V[idx[r, j]] (d bf16 each) into
 * shared memory with 16-byte cp.async (4 warps per CTA, 2-deep per-warp
 * rings, ctas_per_sm CTAs per SM; each chunk's 16 index slots reach a
 * shared ring two chunks before its gather is issued, so no gather waits
 * on an index load), then discards them.  Timing it with CUDA
 * events gives the random-row gather ceiling (bytes = rows*k*2*d*2) that
 * bounds the attention kernel when K/V are resident in L2.
 *   K, V: device bf16 [kv_len, d]; idx: device int32 [rows, k], every entry
 *   in [0, kv_len), 16-byte aligned.  d = 128, k a multiple of 64,
 *   1 <= ctas_per_sm <= 3.
 * Returns IC_OK or IC_ERR_INVALID_ARG / IC_ERR_UNSUPPORTED / IC_ERR_CUDA;
 * asynchronous on `stream`; allocates nothing.
 *
 * ic_probe_wait_timeout is a test aid for failure detection: it enqueues one
 * CTA that waits on a shared-memory barrier nothing ever arrives at, with the
 * same bounded wait the library's pipelined kernels use.  The wait gives up
 * after its limit (about one second), the kernel returns normally and the
 * timeout is latched in ctx, so the next ic_sync_status(ctx, stream) returns
 * IC_ERR_TIMEOUT and clears it; the context stays usable.  Nothing traps or
 * faults.  Returns IC_OK, IC_ERR_INVALID_ARG (ctx NULL) or IC_ERR_CUDA.
 */
#ifndef INDEXCACHE_PROBE_H
#define INDEXCACHE_PROBE_H

#include <stdint.h>

#include "indexcache.h"

#ifdef __cplusplus
extern "C" {
#endif

int ic_probe_gather(const void *K, const void *V, const int32_t *idx, int rows, int k, int d,
                    int ctas_per_sm, void *stream);

int ic_probe_wait_timeout(ic_ctx *ctx, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* INDEXCACHE_PROBE_H */
