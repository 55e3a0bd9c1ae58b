"""Host-side checks of the C ABI (no GPU needed): each library loads and
exports every symbol its header declares (include/indexcache.h for
libindexcache.so, include/indexcache_probe.h for the separate
libindexcache_probe.so, whose symbols the method's library must not carry),
and its host-only logic (patterns, argument checks) behaves; the pattern
resolution is checked against the oracle's."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MAIN_HEADER = os.path.join(ROOT, "include", "indexcache.h")
PROBE_HEADER = os.path.join(ROOT, "include", "indexcache_probe.h")
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def _lib_path():
    from cross_layer_top_b200 import build
    return build.build()


@pytest.fixture(scope="module")
def ic():
    _lib_path()
    from cross_layer_top_b200 import indexcache
    return indexcache


def declared_symbols(headers=(MAIN_HEADER,)):
    text = "\n".join(open(h).read() for h in headers)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(ic_\w+)\s*\(", text, re.M)))


def test_every_header_belongs_to_a_library():
    assert sorted(HEADERS) == sorted([MAIN_HEADER, PROBE_HEADER])


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ["ic_create_pattern", "ic_index_fp", "ic_index_reuse", "ic_sparse_attn",
                 "ic_run_stack", "ic_index_fp_decode", "ic_topk", "ic_index_score"]:
        assert name in syms


def test_library_exports_every_declared_symbol(ic):
    lib = ctypes.CDLL(ic.LIB_PATH)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing
    # and the binding covers the same set
    assert set(declared_symbols()) <= set(ic.EXPORTED)


def test_probe_library_is_separate(ic):
    from cross_layer_top_b200 import probe
    probe_syms = declared_symbols((PROBE_HEADER,))
    assert probe_syms == ["ic_probe_gather", "ic_probe_wait_timeout"]
    plib = ctypes.CDLL(probe.LIB_PATH)
    assert all(hasattr(plib, s) for s in probe_syms)
    assert set(probe_syms) <= set(probe.EXPORTED)
    # the method's library exports none of the aids
    names = subprocess_nm(ic.LIB_PATH)
    assert not [s for s in probe_syms if s in names]


def subprocess_nm(path):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    return {line.split()[-1] for line in out.splitlines() if line.strip()}


def test_version(ic):
    assert ic.ic_version() >= 100


@pytest.mark.parametrize("c", ["FSSSFSSS", "F", "FFFF", "FSFSFSSSSFSFFFFSFFSSFFSFFFSSFFSSFSSSSFSFFFSFSSF"])
def test_pattern_src_matches_oracle(ic, c):
    p = ic.ic_create_pattern(c)
    assert str(p) == c and len(p) == len(c)
    assert ic.ic_pattern_src(p) == oracle.pattern_src(c).tolist()


@pytest.mark.parametrize("n,r", [(8, 4), (47, 1), (47, 2), (47, 4), (47, 8), (16, 4)])
def test_uniform_pattern_matches_oracle(ic, n, r):
    assert str(ic.ic_pattern_uniform(n, r)) == oracle.pattern_uniform(n, r)


@pytest.mark.parametrize("bad", ["", "SFFF", "FSXS", "fsss"])
def test_pattern_errors(ic, bad):
    with pytest.raises(ic.ICError) as e:
        ic.ic_create_pattern(bad)
    assert e.value.code == ic.IC_ERR_PATTERN


def test_index_reuse_aliases(ic):
    assert ic.ic_index_reuse(0x1000) == 0x1000


def test_ctx_create_without_gpu_fails_cleanly(ic):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(ic.ICError) as e:
        ic.Context(0)
    assert e.value.code == ic.IC_ERR_CUDA
