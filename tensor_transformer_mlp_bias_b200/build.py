"""Builds libmlptp.so in-tree for sm_100a with nvcc.

    python -m tensor_transformer_mlp_bias_b200.build [--verbose]

The library is one translation unit (csrc/mlp_tp.cu) with the CUDA runtime
linked statically, so it loads without a GPU and without libcudart on the
library path; the driver entry points it needs are resolved at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "mlp_tp.cu")
OUT = os.path.join(HERE, "libmlptp.so")
DEPS = [os.path.join(HERE, "csrc", n) for n in ("mlp_tp.cu", "gemm.cuh", "ptx.cuh", "colsum.cuh", "fp8.cuh", "peer.cuh", "peer_reduce.cuh")] + [
    os.path.join(os.path.dirname(HERE), "include", "mlp_tp.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "--cudart", "static",
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force: bool = False, verbose: bool = False, defines=(), out: str = None) -> str:
    """Builds the library; returns its path.  `defines` (e.g.
    ["MLPTP_BOUNDS_CHECK"]) and `out` build a variant at another path (always
    rebuilt) instead of the in-tree library."""
    target = out or OUT
    if out is None and not defines and not force and up_to_date():
        return OUT
    tmp = target + ".tmp"
    cmd = ([nvcc()] + NVCC_FLAGS + ["-D" + d for d in defines] + (["-Xptxas", "-v"] if verbose else []) +
           ["-o", tmp, SRC])
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
