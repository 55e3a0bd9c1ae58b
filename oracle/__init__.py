"""CPU oracle for the IndexCache hot path — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference leg may import this package.  The product path
(``cross_layer_top_b200``) never imports it and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64 accumulation, OpenMP over
rows).  This module only marshals arrays into it and runs the layer loop of
Figure 2 ("IndexCache inference") of the page "IndexCache: Accelerating Sparse
Attention via Cross-Layer Index Reuse":

    for each layer l: if c_l = F: I <- INDEXER_l(X); T <- Top-k(I); cache <- T
                      else:       T <- cache
                      X <- SPARSEATTN(X, T)

Inputs are numpy float32 arrays holding bf16 values (exact) or uint8 FP8
bytes.  Every function here is pinned by tests/test_oracle_pins.py.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)

PATTERN_ERRORS = {1: "bad character", 2: "first layer is not F", 3: "bad length"}


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_pattern_src.argtypes = [ctypes.c_char_p, ctypes.c_int, _i32p]
        L.oracle_pattern_uniform.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_char_p]
        L.oracle_index_scores.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, _i32p, ctypes.c_int, _f64p, ctypes.c_int64]
        L.oracle_index_scores_at.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, _i32p, ctypes.c_int, _f64p,
                                             ctypes.c_int64]
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_double.restype = ctypes.c_double
        L.oracle_decode_scores.argtypes = [_f32p, _f32p, _u8p, _f32p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, _f64p]
        L.oracle_index_scores_fp8.argtypes = [_u8p, _f32p, _u8p, _f32p, _f32p, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, _i32p, ctypes.c_int,
                                              _f64p, ctypes.c_int64]
        L.oracle_topk_row.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, _i32p]
        L.oracle_kth_score.argtypes = [_f64p, ctypes.c_int, ctypes.c_int]
        L.oracle_kth_score.restype = ctypes.c_double
        L.oracle_index_topk_rows.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, _i32p, ctypes.c_int, _i32p]
        L.oracle_sparse_attn_row.argtypes = [_f32p, _f32p, _f32p, _i32p, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_double, _f64p]
        L.oracle_sparse_attn_rows.argtypes = [_f32p, _f32p, _f32p, _i32p, _i32p, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int64, ctypes.c_double, _f64p]
        L.oracle_attn_weight_spread_rows.argtypes = [
            _f32p, _f32p, _f32p, _i32p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_double, _f64p]
        L.oracle_overlap_row.argtypes = [_i32p, _i32p, ctypes.c_int]
        L.oracle_overlap_row.restype = ctypes.c_double
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a, ptype):
    return a.ctypes.data_as(ptype)


# --------------------------------------------------------------------------
# Pattern ("IndexCache: Accelerating Sparse Attention via Cross-Layer Index
# Reuse", method details: c in {F,S}^N, f(l) = max{j<l: c_j=F}, first layer F)
# --------------------------------------------------------------------------
def pattern_src(pattern: str) -> np.ndarray:
    """src[l] = l for F layers, f(l) for S layers. Raises ValueError."""
    n = len(pattern)
    src = np.zeros(max(n, 1), dtype=np.int32)
    rc = lib().oracle_pattern_src(pattern.encode("ascii", "replace"), n, _p(src, _i32p))
    if rc != 0:
        raise ValueError("invalid pattern %r: %s" % (pattern, PATTERN_ERRORS.get(rc, rc)))
    return src[:n]


def pattern_uniform(n: int, r: int) -> str:
    """Uniform interleave (§3.1.1): F at l % r == 0."""
    buf = ctypes.create_string_buffer(n + 1)
    rc = lib().oracle_pattern_uniform(n, r, buf)
    if rc != 0:
        raise ValueError("bad uniform pattern n=%d r=%d" % (n, r))
    return buf.value.decode()


# --------------------------------------------------------------------------
# Indexer score (reading-notes page §2.1) and top-k (summary page notation)
# --------------------------------------------------------------------------
def index_scores(q, k, w, rows=None):
    """Scores I[t, s] for s <= t of the requested rows (default: all).

    q: [L, H, d], k: [L, d], w: [L, H] float32.  Returns float64 [nrows, L]
    with NaN where s > t.
    """
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    w = _c(w, np.float32)
    L, H, d = q.shape
    rows = np.arange(L, dtype=np.int32) if rows is None else _c(rows, np.int32)
    out = np.full((len(rows), L), np.nan, dtype=np.float64)
    lib().oracle_index_scores(_p(q, _f32p), _p(k, _f32p), _p(w, _f32p), L, H, d,
                              _p(rows, _i32p), len(rows), _p(out, _f64p), L)
    return out


def index_scores_at(q_rows, w_rows, k, positions):
    """Scores of sampled rows given compactly: q_rows [R, H, d] and w_rows
    [R, H] belong to query positions `positions` [R]; k is [L, d].  Returns
    float64 [R, max(positions)+1] with NaN where s > t."""
    q_rows = _c(q_rows, np.float32)
    w_rows = _c(w_rows, np.float32)
    k = _c(k, np.float32)
    pos = _c(positions, np.int32)
    R, H, d = q_rows.shape
    L = k.shape[0]
    width = int(pos.max()) + 1 if len(pos) else 0
    out = np.full((R, width), np.nan, dtype=np.float64)
    lib().oracle_index_scores_at(_p(q_rows, _f32p), _p(w_rows, _f32p), _p(k, _f32p), L, H, d,
                                 _p(pos, _i32p), R, _p(out, _f64p), width)
    return out


def e4m3_to_float64(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8)
    f = lib().oracle_e4m3_to_double
    return np.array([f(int(x)) for x in b.ravel()], dtype=np.float64).reshape(b.shape)


def decode_scores(q, w, kq, kscale, S=None):
    """Decode-step scores of one sequence: q [H, d], w [H], kq uint8 [S, d]
    (FP8 e4m3 bytes), kscale [S].  Returns float64 [S]."""
    q = _c(q, np.float32)
    w = _c(w, np.float32)
    kq = _c(kq, np.uint8)
    kscale = _c(kscale, np.float32)
    H, d = q.shape
    S = kq.shape[0] if S is None else S
    out = np.empty(S, dtype=np.float64)
    lib().oracle_decode_scores(_p(q, _f32p), _p(w, _f32p), _p(kq, _u8p), _p(kscale, _f32p),
                               S, H, d, _p(out, _f64p))
    return out


def index_scores_fp8(q8, q_scale, k8, k_scale, w, rows=None):
    """FP8 prefill scores (IndexCache paper §2.1, FP8 indexer) on the
    dequantised inputs: q8 uint8 [L, H, d] e4m3 bytes with q_scale [L, H],
    k8 uint8 [L, d] with k_scale [L], w [L, H].  Returns float64
    [nrows, L] with NaN where s > t."""
    q8 = _c(q8, np.uint8)
    k8 = _c(k8, np.uint8)
    q_scale = _c(q_scale, np.float32)
    k_scale = _c(k_scale, np.float32)
    w = _c(w, np.float32)
    L, H, d = q8.shape
    rows = np.arange(L, dtype=np.int32) if rows is None else _c(rows, np.int32)
    out = np.full((len(rows), L), np.nan, dtype=np.float64)
    lib().oracle_index_scores_fp8(_p(q8, _u8p), _p(q_scale, _f32p), _p(k8, _u8p),
                                  _p(k_scale, _f32p), _p(w, _f32p), L, H, d, _p(rows, _i32p),
                                  len(rows), _p(out, _f64p), L)
    return out


def topk_row(score, k: int) -> np.ndarray:
    """Top-k of one score row: ascending indices, ties to the lower index,
    padded with -1 to length k."""
    score = _c(score, np.float64)
    out = np.empty(k, dtype=np.int32)
    lib().oracle_topk_row(_p(score, _f64p), len(score), k, _p(out, _i32p))
    return out


def kth_score(score, k: int) -> float:
    score = _c(score, np.float64)
    return lib().oracle_kth_score(_p(score, _f64p), len(score), k)


def index_topk(q, k, w, topk: int, rows=None) -> np.ndarray:
    """F-layer index rows [nrows, topk] for a prefill layer."""
    q = _c(q, np.float32)
    k = _c(k, np.float32)
    w = _c(w, np.float32)
    L, H, d = q.shape
    rows = np.arange(L, dtype=np.int32) if rows is None else _c(rows, np.int32)
    out = np.empty((len(rows), topk), dtype=np.int32)
    lib().oracle_index_topk_rows(_p(q, _f32p), _p(k, _f32p), _p(w, _f32p), L, H, d, topk,
                                 _p(rows, _i32p), len(rows), _p(out, _i32p))
    return out


# --------------------------------------------------------------------------
# Sparse attention (reading-notes page §3)
# --------------------------------------------------------------------------
def sparse_attn(Q, K, V, idx, rows=None, scale=None, rows_per_seq=0, q_is_rows=False):
    """o[r, h] for the requested rows.  Q: [R, Hq, d] (indexed by row id),
    K, V: [S, d] (one sequence) or [B, S, d] with rows_per_seq rows per
    sequence; idx: [nrows, k] index rows matching ``rows``.  With
    q_is_rows, Q holds only the requested rows, in order.  float64 out."""
    if q_is_rows:
        # attention of row r depends on its own query only: evaluate each
        # requested row as row 0 of a one-row problem over the same K/V
        Q = _c(Q, np.float32)
        out = np.empty((Q.shape[0],) + Q.shape[1:], dtype=np.float64)
        seqs = np.zeros(len(rows), np.int64) if rows_per_seq <= 0 else np.asarray(rows) // rows_per_seq
        for r in range(Q.shape[0]):
            Kr = K if K.ndim == 2 else K[seqs[r]]
            Vr = V if V.ndim == 2 else V[seqs[r]]
            out[r] = sparse_attn(Q[r:r + 1], Kr, Vr, np.asarray(idx)[r:r + 1], scale=scale)[0]
        return out
    Q = _c(Q, np.float32)
    K = _c(K, np.float32)
    V = _c(V, np.float32)
    idx = _c(idx, np.int32)
    R, Hq, d = Q.shape
    rows = np.arange(R, dtype=np.int32) if rows is None else _c(rows, np.int32)
    k = idx.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kv_stride = K.shape[-2] * d if K.ndim == 3 else 0
    out = np.empty((len(rows), Hq, d), dtype=np.float64)
    lib().oracle_sparse_attn_rows(_p(Q, _f32p), _p(K, _f32p), _p(V, _f32p), _p(idx, _i32p),
                                  _p(rows, _i32p), len(rows), k, Hq, d, rows_per_seq,
                                  kv_stride, float(scale), _p(out, _f64p))
    return out


def attn_weight_spread(Q, K, V, idx, rows=None, scale=None, rows_per_seq=0, q_is_rows=False):
    """sqrt(sum_s p_s^2 V[s]^2) per output element, with the softmax weights
    p_s of ``sparse_attn`` (same arguments): how far o moves when every
    weight carries a small independent relative error (the tolerance of the
    attention tests, not a step of the method).  float64 [nrows, Hq, d]."""
    if q_is_rows:
        Q = _c(Q, np.float32)
        out = np.empty((Q.shape[0],) + Q.shape[1:], dtype=np.float64)
        seqs = np.zeros(len(rows), np.int64) if rows_per_seq <= 0 else np.asarray(rows) // rows_per_seq
        for r in range(Q.shape[0]):
            Kr = K if K.ndim == 2 else K[seqs[r]]
            Vr = V if V.ndim == 2 else V[seqs[r]]
            out[r] = attn_weight_spread(Q[r:r + 1], Kr, Vr, np.asarray(idx)[r:r + 1], scale=scale)[0]
        return out
    Q = _c(Q, np.float32)
    K = _c(K, np.float32)
    V = _c(V, np.float32)
    idx = _c(idx, np.int32)
    R, Hq, d = Q.shape
    rows = np.arange(R, dtype=np.int32) if rows is None else _c(rows, np.int32)
    k = idx.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kv_stride = K.shape[-2] * d if K.ndim == 3 else 0
    out = np.empty((len(rows), Hq, d), dtype=np.float64)
    lib().oracle_attn_weight_spread_rows(_p(Q, _f32p), _p(K, _f32p), _p(V, _f32p), _p(idx, _i32p),
                                         _p(rows, _i32p), len(rows), k, Hq, d, rows_per_seq,
                                         kv_stride, float(scale), _p(out, _f64p))
    return out


def overlap(a, b) -> float:
    """|T_i ∩ T_j| / k for one pair of index rows (summary page, Appendix A)."""
    a = _c(a, np.int32)
    b = _c(b, np.int32)
    return lib().oracle_overlap_row(_p(a, _i32p), _p(b, _i32p), len(a))


# --------------------------------------------------------------------------
# The F/S layer loop (summary page, Figure 2 inference procedure)
# --------------------------------------------------------------------------
def run_stack(pattern: str, layers, topk: int, rows=None):
    """Run the prefill stack on CPU.

    layers: list of dicts with 'Q','K','V' for every layer and 'qI','kI','w'
    for F layers (float32 arrays).  Returns (idx_per_layer, out_per_layer);
    idx_per_layer[l] is the index tensor layer l attended with.
    """
    src = pattern_src(pattern)
    cache = None
    idx_used, outs = [], []
    for l, c in enumerate(pattern):
        if c == "F":
            lay = layers[l]
            cache = index_topk(lay["qI"], lay["kI"], lay["w"], topk, rows)
        else:
            assert src[l] < l  # S layer: reuse the cached tensor of f(l)
        idx_used.append(cache)
        outs.append(sparse_attn(layers[l]["Q"], layers[l]["K"], layers[l]["V"], cache, rows))
    return idx_used, outs
