"""Build libattn_b200.so in-tree with nvcc for sm_100a.

    python -m exact_io_aware_sm_b200.build [--verbose]

The library is a plain C-ABI shared object (see include/attn.h); the CUDA
runtime is linked statically and the driver API is reached through
cudaGetDriverEntryPoint, so the .so loads on a machine without a GPU (only
host-side entry points such as attn_classify work there).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libattn_b200.so")
SOURCES = ["api.cu", "plan.cpp", "prefill_sm100.cu", "prefill_f32.cu", "decode.cu", "decode_noalloc.cu",
           "backward.cu", "key_stats.cu"]
HEADERS = ["kernels.h", "plan.h", "ptx_sm100.cuh", "pdl.cuh", "warp_mma.cuh", "fastmath.cuh", os.path.join("..", "..", "include", "attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [__file__]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not verbose and not needs_build():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libattn_b200.so")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
