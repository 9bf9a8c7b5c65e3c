"""Build the C-ABI shared library ``lib/liboq.so`` for sm_100a with nvcc.

The library links the CUDA runtime statically and reaches the driver API only through
``cudaGetDriverEntryPoint``, so it loads on a machine without a GPU (the exported symbols
can be inspected there) and needs only the driver on a GPU machine.

Usage: ``python -m w4a8_ptq_linear_b200.build [--force] [--verbose]``.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(ROOT, "_build", "obj")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "liboq.so")
# the bounds-checked variant (-DOQ_CHECKED): every table-driven device index is range-checked
# and the first violation is reported through the device error word
OBJ_CHECKED = os.path.join(ROOT, "_build", "obj_checked")
LIB_CHECKED = os.path.join(LIB_DIR, "liboq_checked.so")

SOURCES = ["oq_api.cu", "k_rotate_quant.cu", "k_gemm.cu", "k_weights_g64.cu", "oq_plan.cpp",
           "oq_static_scratch.cu", "k_peak.cu", "k_linear_fused.cu"]
HEADERS = ["oq_internal.h", "ptx.cuh", "rq_device.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _flags():
    return ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3",
                   "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                   "--expt-relaxed-constexpr"]


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps += [os.path.join(ROOT, "include", "oq.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra=None, checked: bool = False) -> str:
    """Compile every source to an object, then link lib/liboq.so (lib/liboq_checked.so with
    checked=True). Returns the .so path."""
    LIB, OBJ = (LIB_CHECKED, OBJ_CHECKED) if checked else (globals()["LIB"], globals()["OBJ"])
    if not force and not _stale(LIB):
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    cc = nvcc()
    extra = list(extra or []) + (["-DOQ_CHECKED"] if checked else [])

    def compile_one(src):
        obj = os.path.join(OBJ, os.path.splitext(src)[0] + ".o")
        cmd = [cc] + _flags() + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        return obj

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = LIB + ".tmp"
    cmd = [cc] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs + ["-lpthread"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage")
    ap.add_argument("--checked", action="store_true", help="the bounds-checked variant")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_v else []
    print(build(force=a.force or a.ptxas_v, verbose=a.verbose or a.ptxas_v, extra=extra,
                checked=a.checked))
    sys.exit(0)
