"""cross_layer_top_b200 — B200-native IndexCache hot path.

The compute lives in ``libindexcache.so`` (CUDA for sm_100a behind a C ABI,
declared in ``include/indexcache.h``).  ``cross_layer_top_b200.indexcache``
is the thin ctypes binding with the same names; importing it loads the
library and raises if it is missing.  ``cross_layer_top_b200.synth`` draws
the seeded synthetic inputs.
"""
__all__ = ["indexcache", "synth"]
