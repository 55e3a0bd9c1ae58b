"""Build libindexcache.so (CUDA for sm_100a) in-tree with nvcc.

Each csrc/*.cu is compiled to an object file under _build/ (in parallel) and
linked into cross_layer_top_b200/libindexcache.so with the static CUDA
runtime.  The measurement and test aids in csrc/probe/ become a separate
library, libindexcache_probe.so, linked against libindexcache.so.
``python -m cross_layer_top_b200.build`` or ``build()``.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libindexcache.so")
PROBE_DIR = os.path.join(CSRC, "probe")
PROBE_LIB = os.path.join(HERE, "libindexcache_probe.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libindexcache")
    return exe


def sources(folder=CSRC):
    return sorted(os.path.join(folder, f) for f in os.listdir(folder) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hs + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def _obj(src: str) -> str:
    sub = "probe_" if os.path.dirname(src) == PROBE_DIR else ""
    return os.path.join(OBJ, sub + os.path.basename(src)[:-3] + ".o")


def _compile(src: str, verbose_ptxas: bool) -> str:
    obj = _obj(src)
    newest_dep = max(os.path.getmtime(p) for p in headers() + [src])
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest_dep and not verbose_ptxas:
        return obj
    cmd = [nvcc()] + ARCH + FLAGS + (["-Xptxas", "-v"] if verbose_ptxas else []) + \
        ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def _link(lib: str, objs, extra=()) -> None:
    deps = list(objs) + [p for p in extra if p.endswith(".so")]
    if os.path.exists(lib) and max(os.path.getmtime(o) for o in deps) <= os.path.getmtime(lib):
        return
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + list(objs)
    if extra:
        cmd += ["-L", HERE, "-lindexcache", "-Xlinker", "-rpath,$ORIGIN"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    srcs = sources()
    probe_srcs = sources(PROBE_DIR)
    if force:
        for s in srcs + probe_srcs:
            if os.path.exists(_obj(s)):
                os.remove(_obj(s))
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas), srcs + probe_srcs))
    _link(LIB, objs[:len(srcs)])
    _link(PROBE_LIB, objs[len(srcs):], extra=[LIB])
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
