"""Builds the CUDA library libtsp_b200.so in-tree for sm_100a with nvcc.

    python -m folded_tensor_sequence_rank_b200.build [--verbose]

One translation unit (csrc/tsp_api.cu includes the kernels).  The CUDA
runtime is linked statically; the driver's tensor-map encoder is looked up
at run time, so the library needs no -lcuda.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "tsp_api.cu")
OUT = os.path.join(HERE, "libtsp_b200.so")
# The same source with -DTSP_DEBUG: device index checks that record a status
# (TSP_ERR_BOUNDS) and skip the access instead of faulting.
OUT_DEBUG = os.path.join(HERE, "libtsp_b200_debug.so")
HEADERS = [os.path.join(HERE, "csrc", f) for f in ("ptx.cuh", "gemm_sm100.cuh", "gemm_pair_sm100.cuh", "attn_sm100.cuh",
                                                   "attn_bwd_sm100.cuh", "misc_kernels.cuh")]
HEADERS.append(os.path.join(ROOT, "include", "tsp.h"))


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = OUT, extra=()) -> list:
    return [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
        "-I", os.path.join(ROOT, "include"), *extra, "-o", out, SRC,
    ]


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(f) <= t for f in [SRC, *HEADERS])


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    out = OUT_DEBUG if debug else OUT
    if debug:
        extra = ["-DTSP_DEBUG", *extra]
    if not force and not (extra and not debug) and up_to_date(out):
        return out
    cmd = command(out=out, extra=list(extra))
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stdout.write(res.stdout)
        sys.stderr.write(res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    return out


if __name__ == "__main__":
    v = "--verbose" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build(force=True, verbose=v, extra=extra, debug="--debug" in sys.argv))
