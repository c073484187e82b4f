"""Build liblkv.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python latent_kv_cache_split_b200/build.py [--verbose]

The library is three translation units: csrc/lkv_api.cu (the decode path; it includes the kernel
headers), csrc/lkv_proj.cu (the projections, on the tensor-core GEMM of csrc/lkv_gemm.cuh) and
csrc/lkv_fp8.cu (FP8 latent cache rows).  All link the static CUDA runtime, so the .so only needs
the NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "liblkv.so")
SOURCES = ["lkv_api.cu", "lkv_proj.cu", "lkv_fp8.cu"]
HEADERS = ["lkv_ptx.cuh", "lkv_sched.cuh", "lkv_decode_tc.cuh", "lkv_decode_swap.cuh", "lkv_decode_swap_wide.cuh", "lkv_mla_pair.cuh", "lkv_gemm.cuh", "lkv_aux.cuh", "lkv_tma_host.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC,-O2",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "lkv.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [nvcc_path(), *NVCC_FLAGS]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", LIB + ".tmp"] + [os.path.join(CSRC, s) for s in SOURCES]
    r = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
