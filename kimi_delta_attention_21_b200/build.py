"""Build libkda.so in-tree for sm_100a with nvcc (static CUDA runtime).

    python -m kimi_delta_attention_21_b200.build [--verbose-ptxas] [--checked]

Each csrc/*.cu compiles to _build/<name>.o in parallel, then links into
kimi_delta_attention_21_b200/libkda.so.  Objects are rebuilt when their source
or any header changed.  --checked builds the bounds-checked variant
(-DKDA_CHECKED) from _build_checked/ into libkda_checked.so: every global write
through an offset the library computes is tested against its buffer and, if it
would leave it, skipped and counted (kda_device_bounds_errors).  The binding
loads it when KDA_LIBRARY names it.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkda.so")
BUILD_CHECKED = os.path.join(ROOT, "_build_checked")
LIB_CHECKED = os.path.join(PKG, "libkda_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE, "-I", CSRC,
          "--expt-relaxed-constexpr"]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(obj, deps):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, ptxas_verbose, build_dir=BUILD, extra=()):
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    if not _stale(obj, [src] + _headers()) and not ptxas_verbose:
        return obj, ""
    cmd = [NVCC, *ARCH, *CFLAGS, *extra, "-c", src, "-o", obj + ".tmp"]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    os.replace(obj + ".tmp", obj)
    return obj, r.stderr


def build(ptxas_verbose: bool = False, quiet: bool = True, checked: bool = False) -> str:
    build_dir, lib = (BUILD_CHECKED, LIB_CHECKED) if checked else (BUILD, LIB)
    extra = ("-DKDA_CHECKED",) if checked else ()
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, ptxas_verbose, build_dir, extra), srcs))
    objs = [o for o, _ in results]
    if ptxas_verbose or not quiet:
        for _, log in results:
            if log:
                sys.stderr.write(log)
    if _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(ptxas_verbose="--verbose-ptxas" in sys.argv, quiet=False, checked="--checked" in sys.argv))
