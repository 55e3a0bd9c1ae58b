/*
 * indexcache_probe.h — measurement aid of libindexcache.so (not part of the
 * IndexCache method; the pages have no counterpart).
 *
 * ic_probe_gather enqueues a kernel that performs exactly the K/V row
 * gather of sparse attention and nothing else: for each of `rows` query
 * rows it copies the k rows K[idx[r, j]], V[idx[r, j]] (d bf16 each) into
 * shared memory with 16-byte cp.async (4 warps per CTA, 2-deep per-warp
 * rings, ctas_per_sm CTAs per SM), then discards them.  Timing it with CUDA
 * events gives the random-row gather ceiling (bytes = rows*k*2*d*2) that
 * bounds the attention kernel when K/V are resident in L2.
 *   K, V: device bf16 [kv_len, d]; idx: device int32 [rows, k], every entry
 *   in [0, kv_len).  d = 128, k a multiple of 64, 1 <= ctas_per_sm <= 3.
 * Returns IC_OK or IC_ERR_INVALID_ARG / IC_ERR_UNSUPPORTED / IC_ERR_CUDA;
 * asynchronous on `stream`; allocates nothing.
 */
#ifndef INDEXCACHE_PROBE_H
#define INDEXCACHE_PROBE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int ic_probe_gather(const void *K, const void *V, const int32_t *idx, int rows, int k, int d,
                    int ctas_per_sm, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* INDEXCACHE_PROBE_H */
