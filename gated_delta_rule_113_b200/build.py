"""Build ``libkda.so`` (the C-ABI KDA library) in-tree with nvcc for sm_100a.

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (rebuilt when
it or any header is newer), then linked into ``libkda.so`` next to this file.
The CUDA runtime is linked statically; the driver API (tensor-map encoding)
is reached at run time through ``cudaGetDriverEntryPoint``, so loading the
library needs no ``libcuda`` (it loads on a machine without a GPU).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build", "kda")
LIB = os.path.join(PKG, "libkda.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills",
                     f"-I{INCLUDE}", f"-I{CSRC}"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


# The bounds-checking variant (-DKDA_DEBUG_BOUNDS): every checked global
# index that would leave its buffer is skipped and recorded as KDA_ERR_BOUNDS
# in the device status word; a test build, not the product path.
LIB_DEBUG_BOUNDS = os.path.join(PKG, "libkda_debug_bounds.so")


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug_bounds=False) -> str:
    build_dir = BUILD_DIR + ("_debug_bounds" if debug_bounds else "")
    lib = LIB_DEBUG_BOUNDS if debug_bounds else LIB
    if debug_bounds:
        extra_flags = tuple(extra_flags) + ("-DKDA_DEBUG_BOUNDS",)
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_time = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    nvcc = _nvcc()

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_time)):
            return obj, False
        cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, file=sys.stderr)
        return obj, True

    with ThreadPoolExecutor(max_workers=min(8, len(srcs) or 1)) as ex:
        results = list(ex.map(compile_one, srcs))
    objs = [o for o, _ in results]
    changed = any(c for _, c in results)
    if force or changed or not os.path.exists(lib) or \
            os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build(force="--force" in sys.argv, verbose=True, debug_bounds=True))
