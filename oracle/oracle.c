/*
 * Plain CPU oracle for the IndexCache hot path.  TEST INFRASTRUCTURE ONLY:
 * only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may
 * load this library.  It shares no code, header, table or helper with the
 * CUDA path in cross_layer_top_b200/csrc.
 *
 * Everything is computed in double precision, straight from the definitions,
 * with no blocking, fusion or reordering beyond what the definitions state.
 * Inputs are float arrays holding bf16 values (exact in float) or raw FP8
 * e4m3 bytes; the caller converts.
 *
 * Sources (web pages; cited by title and section):
 *   [IC]  "IndexCache: Accelerating Sparse Attention via Cross-Layer Index
 *          Reuse" (paper summary page): method details (notation, the F/S
 *          pattern c, f(l) = max{j<l : c_j = F}, first layer is F),
 *          Figure 2 inference procedure, §2.1 DSA background (top-k, k=2048).
 *   [RN]  "IndexCache：跨层复用稀疏索引，以及它为什么能被训练" (reading
 *          notes page): §2.1 lightning-indexer score
 *          I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]); §2.2 F/S table and
 *          the FSSS FSSS walk-through (the cache is the current index tensor,
 *          overwritten at the next F); §3 sparse attention
 *          o_t = sum_{s in T_t} softmax(Q_t.K_s / sqrt(d)) V_s.
 *
 * Readings taken where the pages are silent:
 *   causal range s <= t; ties in top-k go to the lower index; the selected
 *   set is returned in ascending index order, padded with -1 when the row
 *   has fewer than k candidates; -1 entries are skipped by attention.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_CHAR 1
#define ORC_FIRST_NOT_F 2
#define ORC_BAD_LEN 3

/* ------------------------------------------------------------------------
 * Pattern: [IC] method details.  c_l in {F,S}; an S layer reuses the index
 * set of f(l) = max{j < l : c_j = F}; the first layer is always F.
 * src[l] = l for an F layer, f(l) for an S layer (0-based).
 * ---------------------------------------------------------------------- */
int oracle_pattern_src(const char *c, int n, int32_t *src)
{
    if (n <= 0)
        return ORC_BAD_LEN;
    for (int l = 0; l < n; ++l)
        if (c[l] != 'F' && c[l] != 'S')
            return ORC_BAD_CHAR;
    if (c[0] != 'F')
        return ORC_FIRST_NOT_F;
    for (int l = 0; l < n; ++l) {
        if (c[l] == 'F') {
            src[l] = l;
        } else {
            /* f(l): the largest j < l with c_j = F, found by scanning back */
            int j = l - 1;
            while (c[j] != 'F')
                --j;
            src[l] = j;
        }
    }
    return ORC_OK;
}

/* Uniform interleave ([IC] §3.1.1): keep the indexer of every r-th layer,
 * i.e. layer l is F iff l % r == 0 (FSSSFSSS... for r = 4). */
int oracle_pattern_uniform(int n, int r, char *out)
{
    if (n <= 0 || r <= 0)
        return ORC_BAD_LEN;
    for (int l = 0; l < n; ++l)
        out[l] = (l % r == 0) ? 'F' : 'S';
    return ORC_OK;
}

/* ------------------------------------------------------------------------
 * Lightning-indexer score, [RN] §2.1:
 *   I[t,s] = sum_{j=1..H} w[t,j] * ReLU( q_I[t,j] . k_I[s] )
 * q: [L, H, d], k: [L, d], w: [L, H].  For each requested row t the scores
 * of s = 0..t are written to out[r*ld + s]; entries s > t are left alone.
 * ---------------------------------------------------------------------- */
static double score_one(const float *q_t, const float *k_s, const float *w_t, int H, int d)
{
    double total = 0.0;
    for (int j = 0; j < H; ++j) {
        const float *qj = q_t + (size_t)j * d;
        double dot = 0.0;
        for (int e = 0; e < d; ++e)
            dot += (double)qj[e] * (double)k_s[e];
        double relu = dot > 0.0 ? dot : 0.0;
        total += (double)w_t[j] * relu;
    }
    return total;
}

void oracle_index_scores(const float *q, const float *k, const float *w, int L, int H, int d,
                         const int32_t *rows, int nrows, double *out, int64_t ld)
{
    int r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; ++r) {
        int t = rows[r];
        if (t < 0 || t >= L)
            continue;
        const float *q_t = q + (size_t)t * H * d;
        const float *w_t = w + (size_t)t * H;
        for (int s = 0; s <= t; ++s)
            out[(size_t)r * ld + s] = score_one(q_t, k + (size_t)s * d, w_t, H, d);
    }
}

/* Same scores for sampled rows whose query tensors are passed compactly:
 * row r has position pos[r], query q_rows[r] ([H, d]) and weights
 * w_rows[r] ([H]); keys k are the whole [L, d] tensor. */
void oracle_index_scores_at(const float *q_rows, const float *w_rows, const float *k, int L, int H,
                            int d, const int32_t *pos, int nrows, double *out, int64_t ld)
{
    int r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; ++r) {
        int t = pos[r];
        if (t < 0 || t >= L)
            continue;
        for (int s = 0; s <= t; ++s)
            out[(size_t)r * ld + s] =
                score_one(q_rows + (size_t)r * H * d, k + (size_t)s * d, w_rows + (size_t)r * H, H, d);
    }
}

/* ------------------------------------------------------------------------
 * OCP FP8 E4M3 decode (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent 0 is subnormal; S.1111.111 is NaN; no infinities).
 * ---------------------------------------------------------------------- */
double oracle_e4m3_to_double(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 15;
    int m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Decode-step score for one sequence (the same [RN] §2.1 formula with one
 * query): the key of candidate s is the dequantised FP8 row
 * k[s,e] = e4m3(kq[s,e]) * scale[s].  out[s] for s = 0..S-1. */
void oracle_decode_scores(const float *q, const float *w, const uint8_t *kq, const float *kscale,
                          int S, int H, int d, double *out)
{
    int s;
#pragma omp parallel for schedule(static)
    for (s = 0; s < S; ++s) {
        double kd[1024];
        for (int e = 0; e < d; ++e)
            kd[e] = oracle_e4m3_to_double(kq[(size_t)s * d + e]) * (double)kscale[s];
        double total = 0.0;
        for (int j = 0; j < H; ++j) {
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += (double)q[(size_t)j * d + e] * kd[e];
            total += (double)w[j] * (dot > 0.0 ? dot : 0.0);
        }
        out[s] = total;
    }
}

/* FP8 prefill scores ([IC] §2.1: the lightning indexer in FP8): the [RN]
 * §2.1 score on the dequantised inputs
 *   q[t,j,e] = e4m3(q8[t,j,e]) * q_scale[t,j],  k[s,e] = e4m3(k8[s,e]) * k_scale[s],
 * everything in double.  Query rows rows[r] (0 <= rows[r] < L); out[r*ld + s]
 * for s <= rows[r].  d <= 1024. */
void oracle_index_scores_fp8(const uint8_t *q8, const float *q_scale, const uint8_t *k8,
                             const float *k_scale, const float *w, int L, int H, int d,
                             const int32_t *rows, int nrows, double *out, int64_t ld)
{
    int r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; ++r) {
        int t = rows[r];
        if (t < 0 || t >= L)
            continue;
        double *qd = (double *)malloc(sizeof(double) * (size_t)H * d);
        for (int j = 0; j < H; ++j)
            for (int e = 0; e < d; ++e)
                qd[(size_t)j * d + e] = oracle_e4m3_to_double(q8[((size_t)t * H + j) * d + e]) *
                                        (double)q_scale[(size_t)t * H + j];
        for (int s = 0; s <= t; ++s) {
            double kd[1024];
            for (int e = 0; e < d; ++e)
                kd[e] = oracle_e4m3_to_double(k8[(size_t)s * d + e]) * (double)k_scale[s];
            double total = 0.0;
            for (int j = 0; j < H; ++j) {
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += qd[(size_t)j * d + e] * kd[e];
                total += (double)w[(size_t)t * H + j] * (dot > 0.0 ? dot : 0.0);
            }
            out[(size_t)r * ld + s] = total;
        }
        free(qd);
    }
}

/* ------------------------------------------------------------------------
 * Top-k ([IC] notation: T_t = Top-k(I_t), k = 2048): full sort of the n
 * candidates by (score descending, index ascending), keep the first
 * min(k, n), return them in ascending index order, pad with -1 to k.
 * ---------------------------------------------------------------------- */
typedef struct {
    double v;
    int32_t i;
} orc_pair;

static int cmp_pair_desc(const void *a, const void *b)
{
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->v > y->v)
        return -1;
    if (x->v < y->v)
        return 1;
    return (x->i > y->i) - (x->i < y->i);
}

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

void oracle_topk_row(const double *score, int n, int k, int32_t *out)
{
    orc_pair *p = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
    for (int s = 0; s < n; ++s) {
        p[s].v = score[s];
        p[s].i = s;
    }
    qsort(p, (size_t)n, sizeof(orc_pair), cmp_pair_desc);
    int m = n < k ? n : k;
    for (int r = 0; r < m; ++r)
        out[r] = p[r].i;
    qsort(out, (size_t)m, sizeof(int32_t), cmp_i32);
    for (int r = m; r < k; ++r)
        out[r] = -1;
    free(p);
}

/* The k-th largest score of a row (the selection threshold), used by the
 * tolerance check on floating-point inputs.  Returns -inf for n < k. */
double oracle_kth_score(const double *score, int n, int k)
{
    if (n < k || k <= 0)
        return -INFINITY;
    orc_pair *p = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)n);
    for (int s = 0; s < n; ++s) {
        p[s].v = score[s];
        p[s].i = s;
    }
    qsort(p, (size_t)n, sizeof(orc_pair), cmp_pair_desc);
    double kth = p[k - 1].v;
    free(p);
    return kth;
}

/* Prefill F layer for a list of rows: scores of s <= t, then top-k.
 * idx_out: [nrows, k]. */
void oracle_index_topk_rows(const float *q, const float *k, const float *w, int L, int H, int d,
                            int topk, const int32_t *rows, int nrows, int32_t *idx_out)
{
    int r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nrows; ++r) {
        int t = rows[r];
        double *row = (double *)malloc(sizeof(double) * (size_t)(t + 1));
        const float *q_t = q + (size_t)t * H * d;
        const float *w_t = w + (size_t)t * H;
        for (int s = 0; s <= t; ++s)
            row[s] = score_one(q_t, k + (size_t)s * d, w_t, H, d);
        oracle_topk_row(row, t + 1, topk, idx_out + (size_t)r * topk);
        free(row);
    }
}

/* ------------------------------------------------------------------------
 * Sparse attention for one query row, [RN] §3:
 *   o[h] = sum_{s in T} softmax_{s in T}( Q[h].K[s] * scale ) V[s]
 * with one shared K/V head (MQA).  idx entries < 0 are skipped.
 * Q: [Hq, d]; K, V: [S, d]; out: [Hq, d].
 * ---------------------------------------------------------------------- */
void oracle_sparse_attn_row(const float *Q, const float *K, const float *V, const int32_t *idx,
                            int k, int Hq, int d, double scale, double *out)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    for (int h = 0; h < Hq; ++h) {
        const float *qh = Q + (size_t)h * d;
        double zmax = -INFINITY;
        for (int r = 0; r < k; ++r) {
            if (idx[r] < 0)
                continue;
            const float *ks = K + (size_t)idx[r] * d;
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += (double)qh[e] * (double)ks[e];
            z[r] = dot * scale;
            if (z[r] > zmax)
                zmax = z[r];
        }
        double denom = 0.0;
        for (int r = 0; r < k; ++r)
            if (idx[r] >= 0)
                denom += exp(z[r] - zmax);
        double *oh = out + (size_t)h * d;
        for (int e = 0; e < d; ++e)
            oh[e] = 0.0;
        for (int r = 0; r < k; ++r) {
            if (idx[r] < 0)
                continue;
            double p = exp(z[r] - zmax) / denom;
            const float *vs = V + (size_t)idx[r] * d;
            for (int e = 0; e < d; ++e)
                oh[e] += p * (double)vs[e];
        }
    }
    free(z);
}

/* Batched form: query row r uses Q + rows[r]*Hq*d, idx + r*k and the K/V
 * block of its sequence, seq = rows[r] / rows_per_seq, at K + seq*kv_stride.
 * out: [nrows, Hq, d]. */
void oracle_sparse_attn_rows(const float *Q, const float *K, const float *V, const int32_t *idx,
                             const int32_t *rows, int nrows, int k, int Hq, int d, int rows_per_seq,
                             int64_t kv_stride, double scale, double *out)
{
    int r;
#pragma omp parallel for schedule(dynamic, 4)
    for (r = 0; r < nrows; ++r) {
        int t = rows[r];
        int64_t seq = rows_per_seq > 0 ? (int64_t)(t / rows_per_seq) : 0;
        oracle_sparse_attn_row(Q + (size_t)t * Hq * d, K + seq * kv_stride, V + seq * kv_stride,
                               idx + (size_t)r * k, k, Hq, d, scale, out + (size_t)r * Hq * d);
    }
}

/* The spread of one attention output under small relative errors in the
 * softmax weights, for the tolerance of the attention tests (not a step of
 * the method).  With the normalised weights p_s of [RN] §3 (the same logits
 * and skipping rule as oracle_sparse_attn_row),
 *   spread[h,e] = sqrt( sum_{s in T} p_s^2 V[s,e]^2 ).
 * If every weight carries an independent relative error of standard
 * deviation u, o[h,e] moves by a random amount of standard deviation
 * u * spread[h,e].  Same argument layout as oracle_sparse_attn_rows. */
void oracle_attn_weight_spread_rows(const float *Q, const float *K, const float *V,
                                    const int32_t *idx, const int32_t *rows, int nrows, int k,
                                    int Hq, int d, int rows_per_seq, int64_t kv_stride,
                                    double scale, double *out)
{
    int r;
#pragma omp parallel for schedule(dynamic, 4)
    for (r = 0; r < nrows; ++r) {
        int t = rows[r];
        int64_t seq = rows_per_seq > 0 ? (int64_t)(t / rows_per_seq) : 0;
        const float *Qt = Q + (size_t)t * Hq * d;
        const float *Kb = K + seq * kv_stride;
        const float *Vb = V + seq * kv_stride;
        const int32_t *ix = idx + (size_t)r * k;
        double *z = (double *)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
        for (int h = 0; h < Hq; ++h) {
            double zmax = -INFINITY;
            for (int j = 0; j < k; ++j) {
                if (ix[j] < 0)
                    continue;
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += (double)Qt[(size_t)h * d + e] * (double)Kb[(size_t)ix[j] * d + e];
                z[j] = dot * scale;
                if (z[j] > zmax)
                    zmax = z[j];
            }
            double denom = 0.0;
            for (int j = 0; j < k; ++j)
                if (ix[j] >= 0)
                    denom += exp(z[j] - zmax);
            double *oh = out + ((size_t)r * Hq + h) * d;
            for (int e = 0; e < d; ++e) {
                double acc = 0.0;
                for (int j = 0; j < k; ++j) {
                    if (ix[j] < 0)
                        continue;
                    double p = exp(z[j] - zmax) / denom;
                    double pv = p * (double)Vb[(size_t)ix[j] * d + e];
                    acc += pv * pv;
                }
                oh[e] = sqrt(acc);
            }
        }
        free(z);
    }
}

/* Cross-layer overlap |T_i ∩ T_j| / k of two index rows ([IC] Appendix A);
 * -1 padding never counts. Both rows must be free of repeated indices. */
double oracle_overlap_row(const int32_t *a, const int32_t *b, int k)
{
    int hits = 0;
    for (int x = 0; x < k; ++x) {
        if (a[x] < 0)
            continue;
        for (int y = 0; y < k; ++y)
            if (b[y] == a[x]) {
                ++hits;
                break;
            }
    }
    return (double)hits / (double)k;
}
