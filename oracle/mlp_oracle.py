"""fp64 CPU oracle of the tensor-parallel Transformer MLP block with biases.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import or call this module.  The
CUDA library never calls it and shares no code with it; the only thing the two
sides share is the seeded input generator, which holds none of the block's
arithmetic.

What it computes
----------------
The block is Megatron's Column->Row parallel MLP ("Megatron-LM — 架构与原理",
§4 巧妙之处, item "Column→Row 配对让 MLP 只做一次通信"; "Megatron-LM（英伟达超大模型
训练框架）完整介绍", §二.2 "MLP层：第一个全连接列切分、第二个全连接行切分"):

    Y = sum_i GeLU(X·A_i + a_i)·B_i + b

with A[h,f] split by columns into t blocks A_i, a_i the matching slice of the
bias a[f], B[f,h] split by rows into B_i, and b[h] added once after the shard
sum.  The split is exact in real arithmetic, so the reference for the whole
block is the plain unsharded definition (``forward`` / ``backward``):

    Z  = X·A + a            H = g(Z)            Y = H·B + b
    dG = dY·Bᵀ              dH = dG ⊙ g'(Z)
    dX = dH·Aᵀ   dA = Xᵀ·dH   da = Σ_rows dH   dB = Hᵀ·dY   db = Σ_rows dY

g is GeLU in its tanh form, g(x) = ½x(1 + tanh(√(2/π)(x + 0.044715x³))), the
approximation published with GELU (Hendrycks & Gimpel, 2016).  The pages do
not name the activation; the tanh form is the reading adopted.

``forward_sharded`` / ``backward_sharded`` spell out the per-shard form the
pages describe (copy/reduce conjugate operators, "Megatron-LM — 架构与原理" §4,
item "通信原语的「前向/反向对偶」"): the forward reduce sums the t partial outputs;
the backward of copy sums the t partial input gradients dX_i.  They exist to
pin the partition invariant, not to serve as the parity reference.

``sample_rows`` / ``sample_ffn`` give exact fp64 values of the same definition
at chosen token rows and ffn indices, for shapes whose full fp64 pass is too
large for the host.

All inputs are the bf16 tensors the GPU sees, upcast exactly to float64.
Nothing is rounded inside the oracle.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Sequence

import numpy as np

SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)
GELU_CUBIC = 0.044715


def f64(x) -> np.ndarray:
    """Exact upcast of a bf16/fp32 torch tensor or array-like to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# activation
# --------------------------------------------------------------------------
def gelu(x: np.ndarray) -> np.ndarray:
    """tanh-form GeLU, g(x) = 0.5·x·(1 + tanh(c·(x + k·x³)))."""
    u = SQRT_2_OVER_PI * (x + GELU_CUBIC * x ** 3)
    return 0.5 * x * (1.0 + np.tanh(u))


def gelu_grad(x: np.ndarray) -> np.ndarray:
    """Derivative of the tanh-form GeLU.

    g'(x) = ½(1 + tanh u) + ½·x·(1 − tanh² u)·c·(1 + 3k·x²),  u = c(x + k·x³).
    """
    u = SQRT_2_OVER_PI * (x + GELU_CUBIC * x ** 3)
    th = np.tanh(u)
    du = SQRT_2_OVER_PI * (1.0 + 3.0 * GELU_CUBIC * x ** 2)
    return 0.5 * (1.0 + th) + 0.5 * x * (1.0 - th * th) * du


# --------------------------------------------------------------------------
# the unsharded block (the parity reference)
# --------------------------------------------------------------------------
def forward(X, A, a, B, b) -> Dict[str, np.ndarray]:
    """Y, Z, H of the block for X[T,h], A[h,f], a[f], B[f,h], b[h]."""
    X, A, a, B, b = (f64(v) for v in (X, A, a, B, b))
    Z = X @ A + a[None, :]
    H = gelu(Z)
    Y = H @ B + b[None, :]
    return {"Y": Y, "Z": Z, "H": H}


def backward(dY, X, A, a, B) -> Dict[str, np.ndarray]:
    """dX, dA, da, dB, db of the block given the output gradient dY[T,h].

    Z and H are recomputed in fp64 from the inputs (no rounding).
    """
    dY, X, A, a, B = (f64(v) for v in (dY, X, A, a, B))
    Z = X @ A + a[None, :]
    H = gelu(Z)
    dG = dY @ B.T
    dH = dG * gelu_grad(Z)
    return {
        "dX": dH @ A.T,
        "dA": X.T @ dH,
        "da": dH.sum(axis=0),
        "dB": H.T @ dY,
        "db": dY.sum(axis=0),
    }


def full(inp: Dict) -> Dict[str, np.ndarray]:
    """Forward and backward outputs for an input dict from the generator."""
    out = forward(inp["X"], inp["A"], inp["a"], inp["B"], inp["b"])
    out.update(backward(inp["dY"], inp["X"], inp["A"], inp["a"], inp["B"]))
    return out


# --------------------------------------------------------------------------
# the sharded form, as the pages describe it (partition-invariant pin)
# --------------------------------------------------------------------------
def shard_slices(f: int, t: int) -> Sequence[slice]:
    if t < 1 or f % t != 0:
        raise ValueError(f"f={f} is not divisible into t={t} shards")
    fs = f // t
    return [slice(i * fs, (i + 1) * fs) for i in range(t)]


def forward_sharded(X, A, a, B, b, t: int) -> Dict[str, object]:
    """Per-shard forward: ColumnParallelLinear (no gather), GeLU,
    RowParallelLinear (parallel input), then the reduce of the t partials
    and one addition of b."""
    X, A, a, B, b = (f64(v) for v in (X, A, a, B, b))
    partials, Zs, Hs = [], [], []
    for sl in shard_slices(A.shape[1], t):
        Z_i = X @ A[:, sl] + a[None, sl]
        H_i = gelu(Z_i)
        partials.append(H_i @ B[sl, :])
        Zs.append(Z_i)
        Hs.append(H_i)
    Y = partials[0].copy()
    for P_i in partials[1:]:
        Y += P_i
    Y += b[None, :]
    return {"Y": Y, "partials": partials, "Z": np.concatenate(Zs, axis=1),
            "H": np.concatenate(Hs, axis=1)}


def backward_sharded(dY, X, A, a, B, t: int) -> Dict[str, object]:
    """Per-shard backward.  dY reaches every shard unchanged (the reduce's
    backward is the identity); each shard forms dH_i and its own weight
    gradients; dX is the sum of the t partial input gradients (the copy's
    backward)."""
    dY, X, A, a, B = (f64(v) for v in (dY, X, A, a, B))
    dX_parts, dA, da, dB = [], [], [], []
    for sl in shard_slices(A.shape[1], t):
        Z_i = X @ A[:, sl] + a[None, sl]
        H_i = gelu(Z_i)
        dH_i = (dY @ B[sl, :].T) * gelu_grad(Z_i)
        dX_parts.append(dH_i @ A[:, sl].T)
        dA.append(X.T @ dH_i)
        da.append(dH_i.sum(axis=0))
        dB.append(H_i.T @ dY)
    dX = dX_parts[0].copy()
    for Q_i in dX_parts[1:]:
        dX += Q_i
    return {"dX": dX, "dX_partials": dX_parts,
            "dA": np.concatenate(dA, axis=1), "da": np.concatenate(da),
            "dB": np.concatenate(dB, axis=0), "db": dY.sum(axis=0)}


# --------------------------------------------------------------------------
# exact values at sampled indices (large shapes)
# --------------------------------------------------------------------------
def sample_rows(inp: Dict, rows: Iterable[int]) -> Dict[str, np.ndarray]:
    """Exact Y, Z, H, dX at the given token rows (each row of the block is
    independent of the others in the forward and in dX)."""
    rows = np.asarray(list(rows), dtype=np.int64)
    X = f64(inp["X"][rows])
    dY = f64(inp["dY"][rows])
    A, a, B, b = (f64(inp[k]) for k in ("A", "a", "B", "b"))
    Z = X @ A + a[None, :]
    H = gelu(Z)
    Y = H @ B + b[None, :]
    dH = (dY @ B.T) * gelu_grad(Z)
    dX = dH @ A.T
    return {"rows": rows, "Y": Y, "Z": Z, "H": H, "dX": dX}


def sample_ffn(inp: Dict, cols: Iterable[int]) -> Dict[str, np.ndarray]:
    """Exact dA[:, j], da[j], dB[j, :] and db for the given ffn indices j.

    Column j of Z and dH depends only on A[:, j], a[j], B[j, :], X and dY.
    """
    cols = np.asarray(list(cols), dtype=np.int64)
    X = f64(inp["X"])
    dY = f64(inp["dY"])
    A_c = f64(inp["A"][:, cols])
    a_c = f64(inp["a"][cols])
    B_r = f64(inp["B"][cols, :])
    Z = X @ A_c + a_c[None, :]
    H = gelu(Z)
    dH = (dY @ B_r.T) * gelu_grad(Z)
    return {"cols": cols, "dA": X.T @ dH, "da": dH.sum(axis=0),
            "dB": H.T @ dY, "db": dY.sum(axis=0), "Zcol": Z, "Hcol": H}


def flops(T: int, h: int, f: int) -> int:
    """Algorithmic FLOPs of one forward+backward (six GEMMs of 2·T·h·f)."""
    return 12 * T * h * f
