"""ctypes binding of libindexcache_probe.so (include/indexcache_probe.h):
measurement and test aids kept out of the method's library.

ic_probe_gather is the sparse attention's K/V row gather alone (the L2
gather ceiling the benchmark rates attention against);
ic_probe_wait_timeout makes one bounded device wait run out (the
failure-detection test).  Importing this module without the built library
raises ImportError.
"""
from __future__ import annotations

import ctypes
import os

from . import indexcache as _ic

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libindexcache_probe.so")
if not os.path.exists(LIB_PATH):
    raise ImportError("libindexcache_probe.so is not built (run `python -m "
                      "cross_layer_top_b200.build`)")
_lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_SIGS = {
    "ic_probe_gather": ([_vp, _vp, _vp, _i, _i, _i, _i, _vp], _i),
    "ic_probe_wait_timeout": ([_vp, _vp], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = sorted(_SIGS)


def ic_probe_wait_timeout(ctx: "_ic.Context", stream=None):
    """Test aid: one bounded device wait that runs out (about a second); the
    next ctx.sync_status() raises IC_ERR_TIMEOUT."""
    _ic._check(_lib.ic_probe_wait_timeout(ctx.handle, _ic._stream(stream)), ctx)


def ic_probe_gather(K, V, idx, ctas_per_sm: int = 2, stream=None):
    """Measurement aid: the attention's K/V row gather alone (no compute)."""
    rows, k = idx.shape
    _ic._check(_lib.ic_probe_gather(_ic._ptr(K), _ic._ptr(V), _ic._ptr(idx), rows, k,
                                    K.shape[-1], ctas_per_sm, _ic._stream(stream)))
