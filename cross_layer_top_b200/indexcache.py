"""Thin ctypes binding of libindexcache.so (include/indexcache.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels.  Functions carry the C names; tensors are torch tensors on the
context's GPU (their data pointers are passed), streams default to torch's
current stream.  Importing this module loads the library and raises
ImportError when it is missing — there is no fallback path.
"""
from __future__ import annotations

import ctypes
import weakref
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libindexcache.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libindexcache.so is not built (run `python -m cross_layer_top_b200.build`): "
                      "the CUDA library is required, there is no CPU path")
_lib = ctypes.CDLL(LIB_PATH)

IC_OK = 0
IC_ERR_INVALID_ARG = 1
IC_ERR_PATTERN = 2
IC_ERR_SHAPE = 3
IC_ERR_UNSUPPORTED = 4
IC_ERR_CUDA = 5
IC_ERR_TIMEOUT = 6
IC_ERR_NOMEM = 7
IC_ERR_DEVICE = 8
IC_PREFILL = 0
IC_DECODE = 1
IC_K_INDEX_SCORE = 0
IC_K_INDEX_SCORE_DECODE = 1
IC_K_TOPK = 2
IC_K_ATTN = 3
IC_K_OVERLAP = 4
IC_K_COUNT = 5
KERNEL_NAMES = ["index_score", "index_score_decode", "topk", "sparse_attn", "index_overlap"]

_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float


class ic_layer_io(ctypes.Structure):
    _fields_ = [("qI", _vp), ("kI", _vp), ("w", _vp), ("kI8", _vp), ("kI_scale", _vp),
                ("Q", _vp), ("K", _vp), ("V", _vp), ("out", _vp), ("idx_snapshot", _vp)]


class ic_stack_dims(ctypes.Structure):
    _fields_ = [("mode", _i), ("L", _i), ("B", _i), ("S_max", _i), ("seq_len", _vp),
                ("H_I", _i), ("d_I", _i), ("k", _i), ("Hq", _i), ("d", _i), ("scale", _f)]


_SIGS = {
    "ic_version": ([], _i),
    "ic_ctx_create": ([ctypes.POINTER(_vp), _i, ctypes.c_size_t], _i),
    "ic_ctx_destroy": ([_vp], _i),
    "ic_last_error": ([_vp], ctypes.c_char_p),
    "ic_sync_status": ([_vp, _vp], _i),
    "ic_ctx_set_timing": ([_vp, _i], _i),
    "ic_ctx_get_timing": ([_vp, _i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64)], _i),
    "ic_ctx_reset_timing": ([_vp], _i),
    "ic_ctx_launch_count": ([_vp], _i64),
    "ic_create_pattern": ([ctypes.c_char_p, _i, ctypes.POINTER(_vp)], _i),
    "ic_pattern_uniform": ([_i, _i, ctypes.POINTER(_vp)], _i),
    "ic_pattern_destroy": ([_vp], _i),
    "ic_pattern_size": ([_vp], _i),
    "ic_pattern_string": ([_vp, ctypes.c_char_p, _i], _i),
    "ic_pattern_src": ([_vp, ctypes.POINTER(ctypes.c_int32)], _i),
    "ic_index_score": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i64, _vp], _i),
    "ic_topk": ([_vp, _vp, _i64, _i, _i, _i, _vp, _vp, _i64, _vp], _i),
    "ic_index_fp": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp], _i),
    "ic_index_reuse": ([_vp, ctypes.POINTER(_vp)], _i),
    "ic_index_score_decode": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _i64, _vp], _i),
    "ic_index_fp_decode": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp], _i),
    "ic_index_fp_decode_noalloc": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp], _i),
    "ic_sparse_attn": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64, _i, _f, _vp, _vp], _i),
    "ic_index_overlap": ([_vp, _vp, _vp, _i, _i, _i, _vp, _vp], _i),
    "ic_index_score_fp8": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i64, _vp], _i),
    "ic_index_fp_fp8": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp], _i),
    "ic_noalloc_sync_status": ([_vp], _i),
    "ic_run_stack": ([_vp, _vp, ctypes.POINTER(ic_layer_io), ctypes.POINTER(ic_stack_dims), _vp,
                      _vp], _i),
    "ic_run_stack_host": ([_vp, _vp, ctypes.POINTER(ic_layer_io), ctypes.POINTER(ic_stack_dims),
                           _vp, _vp], _i),
    "ic_run_stack_ahead": ([_vp, _vp, ctypes.POINTER(ic_layer_io), ctypes.POINTER(ic_stack_dims),
                            _vp, _vp, _vp], _i),
    "ic_run_stack_rows": ([_vp, _vp, ctypes.POINTER(ic_layer_io), ctypes.POINTER(ic_stack_dims),
                           ctypes.POINTER(ctypes.c_int32), _i, _vp, _vp], _i),
    "ic_prefill_partition": ([_i, _i, _i, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(_i)], _i),
    "ic_index_fp_rows": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp], _i),
    "ic_stack_graph_create": ([_vp, _vp, ctypes.POINTER(ic_layer_io),
                               ctypes.POINTER(ic_stack_dims), _vp, ctypes.POINTER(_vp)], _i),
    "ic_stack_graph_create_ahead": ([_vp, _vp, ctypes.POINTER(ic_layer_io),
                                     ctypes.POINTER(ic_stack_dims), _vp, _vp,
                                     ctypes.POINTER(_vp)], _i),
    "ic_stack_graph_launch": ([_vp, _vp], _i),
    "ic_stack_graph_kernels": ([_vp], _i64),
    "ic_stack_graph_destroy": ([_vp], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = sorted(_SIGS)


class ICError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("libindexcache error %d: %s" % (code, msg))
        self.code = code


def _check(rc, ctx=None):
    if rc != IC_OK:
        msg = _lib.ic_last_error(ctx.handle if ctx is not None else None)
        raise ICError(rc, msg.decode(errors="replace") if msg else "")


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dev_tensor(t, dtype, name):
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


class Context:
    """Owns an ic_ctx (scratch memory, device error word, timing counters)."""

    def __init__(self, device: int = 0, scratch_bytes: int = 0):
        h = _vp()
        _check(_lib.ic_ctx_create(ctypes.byref(h), device, scratch_bytes))
        self.handle = h
        self.device = device
        self._graphs = weakref.WeakSet()

    def close(self):
        for g in list(self._graphs):
            g.close()
        if self.handle:
            _lib.ic_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def sync_status(self, stream=None):
        _check(_lib.ic_sync_status(self.handle, _stream(stream)), self)

    def set_timing(self, enable: bool):
        _check(_lib.ic_ctx_set_timing(self.handle, int(enable)), self)

    def get_timing(self, kernel: int):
        ms = ctypes.c_double()
        n = _i64()
        _check(_lib.ic_ctx_get_timing(self.handle, kernel, ctypes.byref(ms), ctypes.byref(n)), self)
        return ms.value, n.value

    def reset_timing(self):
        _check(_lib.ic_ctx_reset_timing(self.handle), self)

    def launch_count(self) -> int:
        return int(_lib.ic_ctx_launch_count(self.handle))


class Pattern:
    """An F/S layer pattern (ic_pattern)."""

    def __init__(self, c: str | None = None, n_layers: int | None = None, r: int | None = None):
        h = _vp()
        if c is not None:
            b = c.encode("ascii", "replace")
            _check(_lib.ic_create_pattern(b, len(b), ctypes.byref(h)))
        else:
            _check(_lib.ic_pattern_uniform(n_layers, r, ctypes.byref(h)))
        self.handle = h

    def __del__(self):
        try:
            if self.handle:
                _lib.ic_pattern_destroy(self.handle)
                self.handle = None
        except Exception:
            pass

    def __len__(self):
        return _lib.ic_pattern_size(self.handle)

    def __str__(self):
        n = len(self)
        buf = ctypes.create_string_buffer(n + 1)
        _check(_lib.ic_pattern_string(self.handle, buf, n + 1))
        return buf.value.decode()

    def src(self):
        n = len(self)
        arr = (ctypes.c_int32 * n)()
        _check(_lib.ic_pattern_src(self.handle, arr))
        return list(arr)


def ic_version() -> int:
    return _lib.ic_version()


def ic_create_pattern(c: str) -> Pattern:
    return Pattern(c)


def ic_pattern_uniform(n_layers: int, r: int) -> Pattern:
    return Pattern(n_layers=n_layers, r=r)


def ic_pattern_src(p: Pattern):
    return p.src()


def ic_index_score(ctx: Context, qI, kI, w, row_begin: int, row_end: int, scores, ld=None,
                   stream=None):
    L, H_I, d_I = qI.shape
    for t, n in ((qI, "qI"), (kI, "kI"), (w, "w")):
        _dev_tensor(t, torch.bfloat16, n)
    _dev_tensor(scores, torch.float32, "scores")
    ld = scores.shape[-1] if ld is None else ld
    _check(_lib.ic_index_score(ctx.handle, _ptr(qI), _ptr(kI), _ptr(w), L, H_I, d_I, row_begin,
                               row_end, _ptr(scores), ld, _stream(stream)), ctx)


def ic_topk(ctx: Context, scores, k: int, idx_out, causal_base: int = 0, row_len=None,
            rows=None, ld=None, stream=None):
    _dev_tensor(idx_out, torch.int32, "idx_out")
    rows = idx_out.shape[0] if rows is None else rows
    ld = scores.shape[-1] if ld is None else ld
    _check(_lib.ic_topk(ctx.handle, _ptr(scores), ld, rows, k, causal_base, _ptr(row_len),
                        _ptr(idx_out), idx_out.shape[-1], _stream(stream)), ctx)


def ic_index_fp(ctx: Context, qI, kI, w, k: int, idx_out, stream=None):
    L, H_I, d_I = qI.shape
    for t, n in ((qI, "qI"), (kI, "kI"), (w, "w")):
        _dev_tensor(t, torch.bfloat16, n)
    _dev_tensor(idx_out, torch.int32, "idx_out")
    _check(_lib.ic_index_fp(ctx.handle, _ptr(qI), _ptr(kI), _ptr(w), L, H_I, d_I, k,
                            _ptr(idx_out), _stream(stream)), ctx)


def ic_index_reuse(idx_cache):
    out = _vp()
    _check(_lib.ic_index_reuse(_ptr(idx_cache), ctypes.byref(out)))
    return out.value


def ic_index_score_decode(ctx: Context, q, w, kI8, kI_scale, seq_len, scores, ld=None,
                          stream=None):
    B, H_I, d_I = q.shape
    S_max = kI8.shape[1]
    ld = scores.shape[-1] if ld is None else ld
    _check(_lib.ic_index_score_decode(ctx.handle, _ptr(q), _ptr(w), _ptr(kI8), _ptr(kI_scale),
                                      _ptr(seq_len), B, S_max, H_I, d_I, _ptr(scores), ld,
                                      _stream(stream)), ctx)


def ic_index_fp_decode(ctx: Context, q, w, kI8, kI_scale, seq_len, k: int, idx_out, stream=None):
    B, H_I, d_I = q.shape
    S_max = kI8.shape[1]
    _check(_lib.ic_index_fp_decode(ctx.handle, _ptr(q), _ptr(w), _ptr(kI8), _ptr(kI_scale),
                                   _ptr(seq_len), B, S_max, H_I, d_I, k, _ptr(idx_out),
                                   _stream(stream)), ctx)


def ic_index_fp_decode_noalloc(q, w, kI8, kI_scale, seq_len, k: int, idx_out, stream=None):
    """Decode F layer without any device allocation (fixed library scratch)."""
    B, H_I, d_I = q.shape
    S_max = kI8.shape[1]
    _check(_lib.ic_index_fp_decode_noalloc(_ptr(q), _ptr(w), _ptr(kI8), _ptr(kI_scale),
                                           _ptr(seq_len), B, S_max, H_I, d_I, k, _ptr(idx_out),
                                           _stream(stream)))


def ic_noalloc_sync_status(stream=None):
    """Synchronize `stream`, then report (and clear) the device error word of
    the allocation-free path on the current device; raises ICError."""
    _check(_lib.ic_noalloc_sync_status(_stream(stream)))


def ic_sparse_attn(ctx: Context, Q, K, V, idx, out, rows_per_seq: int = 0, kv_seq_stride: int = 0,
                   kv_len=None, scale: float = 0.0, stream=None):
    rows, Hq, d = Q.shape
    k = idx.shape[-1]
    if kv_len is None:
        kv_len = K.shape[-2]
    _check(_lib.ic_sparse_attn(ctx.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(idx), rows, Hq, d, k,
                               rows_per_seq, kv_seq_stride, kv_len, scale, _ptr(out),
                               _stream(stream)), ctx)


def ic_index_score_fp8(ctx: Context, qI8, q_scale, kI8, k_scale, w, row_begin: int, row_end: int,
                       scores, ld=None, stream=None):
    """FP8 indexer scores: qI8 uint8 (e4m3 bytes) [L, H_I, d_I], q_scale f32
    [L, H_I], kI8 uint8 [L, d_I], k_scale f32 [L], w bf16 [L, H_I]."""
    L, H_I, d_I = qI8.shape
    for t, dt, n in ((qI8, torch.uint8, "qI8"), (kI8, torch.uint8, "kI8"),
                     (q_scale, torch.float32, "q_scale"), (k_scale, torch.float32, "k_scale"),
                     (w, torch.bfloat16, "w"), (scores, torch.float32, "scores")):
        _dev_tensor(t, dt, n)
    ld = scores.shape[-1] if ld is None else ld
    _check(_lib.ic_index_score_fp8(ctx.handle, _ptr(qI8), _ptr(q_scale), _ptr(kI8), _ptr(k_scale),
                                   _ptr(w), L, H_I, d_I, row_begin, row_end, _ptr(scores), ld,
                                   _stream(stream)), ctx)


def ic_index_fp_fp8(ctx: Context, qI8, q_scale, kI8, k_scale, w, k: int, idx_out, stream=None):
    """FP8 prefill F layer: scores + top-k into idx_out int32 [L, k]."""
    L, H_I, d_I = qI8.shape
    for t, dt, n in ((qI8, torch.uint8, "qI8"), (kI8, torch.uint8, "kI8"),
                     (q_scale, torch.float32, "q_scale"), (k_scale, torch.float32, "k_scale"),
                     (w, torch.bfloat16, "w"), (idx_out, torch.int32, "idx_out")):
        _dev_tensor(t, dt, n)
    _check(_lib.ic_index_fp_fp8(ctx.handle, _ptr(qI8), _ptr(q_scale), _ptr(kI8), _ptr(k_scale),
                                _ptr(w), L, H_I, d_I, k, _ptr(idx_out), _stream(stream)), ctx)


def ic_index_overlap(ctx: Context, idx_a, idx_b, hits, n_keys: int, stream=None):
    """hits[r] = |T_a[r] ∩ T_b[r]| for two [rows, k] int32 index tensors
    (the overlap of row r is hits[r] / k)."""
    rows, k = idx_a.shape
    if tuple(idx_b.shape) != (rows, k):
        raise ValueError("idx_a and idx_b must have the same shape")
    _check(_lib.ic_index_overlap(ctx.handle, _ptr(idx_a), _ptr(idx_b), rows, k, n_keys, _ptr(hits),
                                 _stream(stream)), ctx)


def make_stack_layers(layers, mode=IC_PREFILL):
    """layers: list of dicts with torch tensors (qI/kI/w or q/w/kI8/kI_scale
    on F layers; Q/K/V/out and optional idx_snapshot on every layer)."""
    arr = (ic_layer_io * len(layers))()
    for l, lay in enumerate(layers):
        io = arr[l]
        io.qI = _ptr(lay.get("qI", lay.get("q")))
        io.kI = _ptr(lay.get("kI"))
        io.w = _ptr(lay.get("w"))
        io.kI8 = _ptr(lay.get("kI8"))
        io.kI_scale = _ptr(lay.get("kI_scale"))
        io.Q = _ptr(lay["Q"])
        io.K = _ptr(lay["K"])
        io.V = _ptr(lay["V"])
        io.out = _ptr(lay["out"])
        io.idx_snapshot = _ptr(lay.get("idx_snapshot"))
    return arr


def ic_run_stack(ctx: Context, pattern: Pattern, layers, dims: ic_stack_dims, idx_cache,
                 stream=None, layer_array=None):
    arr = layer_array if layer_array is not None else make_stack_layers(layers, dims.mode)
    _check(_lib.ic_run_stack(ctx.handle, pattern.handle, arr, ctypes.byref(dims),
                             _ptr(idx_cache), _stream(stream)), ctx)


def ic_run_stack_ahead(ctx: Context, pattern: Pattern, layers, dims: ic_stack_dims, idx_cache,
                       idx_cache2, stream=None, layer_array=None):
    """ic_run_stack with each F layer's indexer issued ahead on a second
    stream; the j-th F layer's indices go to idx_cache (j even) or
    idx_cache2 (j odd)."""
    arr = layer_array if layer_array is not None else make_stack_layers(layers, dims.mode)
    _check(_lib.ic_run_stack_ahead(ctx.handle, pattern.handle, arr, ctypes.byref(dims),
                                   _ptr(idx_cache), _ptr(idx_cache2), _stream(stream)), ctx)


def ic_run_stack_host(ctx: Context, pattern: Pattern, layers_host, dims: ic_stack_dims, idx_cache,
                      stream=None, layer_array=None):
    """ic_run_stack on inputs in (pinned) host memory: layers_host holds CPU
    tensors for every field but idx_snapshot; each layer's 'out' (a CPU
    tensor) receives its output.  Asynchronous on `stream`."""
    if layer_array is None:
        for lay in layers_host:
            for n, t in lay.items():
                if n != "idx_snapshot" and t is not None and t.is_cuda:
                    raise ValueError("%s must be a host tensor" % n)
        layer_array = make_stack_layers(layers_host, dims.mode)
    _check(_lib.ic_run_stack_host(ctx.handle, pattern.handle, layer_array, ctypes.byref(dims),
                                  _ptr(idx_cache), _stream(stream)), ctx)


def ic_prefill_partition(L: int, world: int, rank: int):
    """The rank's query-row ranges [(a0, b0), (a1, b1)] of a causal-balanced
    split of L rows over `world` ranks (host only)."""
    r = (ctypes.c_int32 * 4)()
    n = _i()
    _check(_lib.ic_prefill_partition(L, world, rank, r, ctypes.byref(n)))
    return [(int(r[2 * i]), int(r[2 * i + 1])) for i in range(n.value)]


def ic_index_fp_rows(ctx: Context, qI_rows, w_rows, kI, row_begin: int, row_end: int, k: int,
                     idx_out, stream=None):
    """F layer of rows [row_begin, row_end) with compact q_I / w rows and the
    whole k_I [L, d_I]; idx_out int32 [row_end - row_begin, k]."""
    n, H_I, d_I = qI_rows.shape
    if n != row_end - row_begin:
        raise ValueError("qI_rows must hold row_end - row_begin rows")
    _check(_lib.ic_index_fp_rows(ctx.handle, _ptr(qI_rows), _ptr(w_rows), _ptr(kI), kI.shape[0],
                                 H_I, d_I, row_begin, row_end, k, _ptr(idx_out), _stream(stream)),
           ctx)


def ic_run_stack_rows(ctx: Context, pattern: Pattern, layers, dims: ic_stack_dims, ranges,
                      idx_cache, stream=None, layer_array=None):
    """One rank's share of a prefill stack split by rows: `ranges` are its
    (begin, end) row ranges; qI/w/Q/out (and idx_snapshot) of each layer hold
    those rows only, kI/K/V all L rows."""
    arr = layer_array if layer_array is not None else make_stack_layers(layers, dims.mode)
    flat = (ctypes.c_int32 * (2 * len(ranges)))(*[v for ab in ranges for v in ab])
    _check(_lib.ic_run_stack_rows(ctx.handle, pattern.handle, arr, ctypes.byref(dims), flat,
                                  len(ranges), _ptr(idx_cache), _stream(stream)), ctx)


class StackGraph:
    """ic_stack_graph_*: the stack captured once and replayed.  The graph
    keeps the device addresses of the layer tensors, dims.seq_len and
    idx_cache, so this object holds references to them; change their
    contents in place between launches.  With idx_cache2, the schedule of
    ic_run_stack_ahead is captured (ic_stack_graph_create_ahead)."""

    def __init__(self, ctx: Context, pattern: Pattern, layers, dims: ic_stack_dims, idx_cache,
                 layer_array=None, idx_cache2=None):
        arr = layer_array if layer_array is not None else make_stack_layers(layers, dims.mode)
        h = _vp()
        if idx_cache2 is None:
            rc = _lib.ic_stack_graph_create(ctx.handle, pattern.handle, arr, ctypes.byref(dims),
                                            _ptr(idx_cache), ctypes.byref(h))
        else:
            rc = _lib.ic_stack_graph_create_ahead(ctx.handle, pattern.handle, arr,
                                                  ctypes.byref(dims), _ptr(idx_cache),
                                                  _ptr(idx_cache2), ctypes.byref(h))
        _check(rc, ctx)
        self.handle = h
        self.ctx = ctx
        ctx._graphs.add(self)
        self._keep = (pattern, layers, dims, idx_cache, idx_cache2, arr)

    def launch(self, stream=None):
        _check(_lib.ic_stack_graph_launch(self.handle, _stream(stream)), self.ctx)

    def kernels(self) -> int:
        return int(_lib.ic_stack_graph_kernels(self.handle))

    def close(self):
        if self.handle:
            _lib.ic_stack_graph_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ic_stack_graph_create(ctx: Context, pattern: Pattern, layers, dims: ic_stack_dims, idx_cache,
                          layer_array=None) -> StackGraph:
    return StackGraph(ctx, pattern, layers, dims, idx_cache, layer_array)


def ic_stack_graph_create_ahead(ctx: Context, pattern: Pattern, layers, dims: ic_stack_dims,
                                idx_cache, idx_cache2, layer_array=None) -> StackGraph:
    return StackGraph(ctx, pattern, layers, dims, idx_cache, layer_array, idx_cache2)


def stack_dims(mode, H_I, d_I, k, Hq, d, L=0, B=0, S_max=0, seq_len=None, scale=0.0):
    return ic_stack_dims(mode, L, B, S_max, _ptr(seq_len), H_I, d_I, k, Hq, d, scale)
