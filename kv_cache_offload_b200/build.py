"""Build libdkv.so in-tree for sm_100a with nvcc (no JIT cache, no torch extension).

Each csrc/*.cu and csrc/*.cpp (host-only C++) is compiled to an object under <repo>/_build/
in parallel, then linked into kv_cache_offload_b200/libdkv.so. The same sources compiled
with -DDKV_DEBUG (device-side range checks on every block, slot and workspace index a
kernel computes; failures flag the pool's status word instead of touching memory) are
linked into kv_cache_offload_b200/libdkv_debug.so, which the binding loads when the
environment sets DKV_LIBRARY=debug. Rebuilds only when a source or header is newer than
the library.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdkv.so")
LIB_DEBUG = os.path.join(PKG, "libdkv_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(ROOT, "include", "*.h")) + [os.path.abspath(__file__)])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def _build_one(lib: str, defines, verbose: bool, ptxas_info: bool) -> str:
    nvcc = _nvcc()
    objdir = os.path.join(BUILD, "debug" if defines else "release")
    os.makedirs(objdir, exist_ok=True)
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + list(defines)

    def comp(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        res = list(ex.map(comp, _sources()))
    if verbose or ptxas_info:
        for _, err in res:
            if err:
                sys.stderr.write(err)
    tmp = lib + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp] + [o for o, _ in res] + ["-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug: bool = True) -> str:
    """Build libdkv.so (and, unless debug=False, libdkv_debug.so) if out of date."""
    if force or not up_to_date(LIB):
        _build_one(LIB, [], verbose, ptxas_info)
    if debug and (force or not up_to_date(LIB_DEBUG)):
        _build_one(LIB_DEBUG, ["-DDKV_DEBUG"], verbose, False)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv))
