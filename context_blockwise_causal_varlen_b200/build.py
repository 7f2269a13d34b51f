"""Build libcbv.so in place (nvcc, sm_100a).

Usage: ``python -m context_blockwise_causal_varlen_b200.build [--debug]`` or ``build()``.
Each source compiles to an object under ``_build/`` in parallel, then links into
``context_blockwise_causal_varlen_b200/libcbv.so`` next to this file.  ``debug=True``
builds ``libcbv_debug.so`` instead (objects under ``_build/debug``): the same sources
compiled with ``CBV_DEBUG``, whose kernels check every row and page index against its
tensor before a copy or store and report a violation through the status word.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libcbv.so")
DEBUG_LIB = os.path.join(HERE, "libcbv_debug.so")

SOURCES = ["api.cu", "fwd_pp.cu", "bwd.cu", "cached.cu", "decode.cu", "misc.cu", "noalloc.cu", "plan.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-lineinfo", f"-I{os.path.join(ROOT, 'include')}"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    out_dir = os.path.join(OUT_DIR, "debug") if debug else OUT_DIR
    obj = os.path.join(out_dir, os.path.splitext(src)[0] + ".o")
    path = os.path.join(CSRC, src)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "cbv.h")]
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(d) for d in deps):
        return obj
    cmd = [_nvcc(), *ARCH, *COMMON, *(["-DCBV_DEBUG"] if debug else []), "-c", path, "-o", obj]
    if verbose and src.endswith(".cu"):
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stderr}")
    if verbose:
        sys.stderr.write(res.stderr)
    return obj


def build(verbose: bool = False, debug: bool = False) -> str:
    os.makedirs(os.path.join(OUT_DIR, "debug") if debug else OUT_DIR, exist_ok=True)
    lib = DEBUG_LIB if debug else LIB
    with cf.ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug), SOURCES))
    if not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        cmd = [_nvcc(), *ARCH, "-shared", "-o", lib, *objs, "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stderr}")
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, debug="--debug" in sys.argv))
