"""Precision of the cross-GPU reduction, checked on the CPU.

With the block sharded over N GPUs, each rank computes a partial
P_r = H_r·B_r of Y (and Q_r = dH_r·A_rᵀ of dX), and the partials are summed
across ranks: the forward all-reduce of the reduce operator and the backward
all-reduce of the copy operator ("Megatron-LM — 架构与原理", §4 巧妙之处, item
"通信原语的「前向/反向对偶」").  The pages' system all-reduces the 16-bit
outputs of each rank.  This test emulates both choices in fp64 at sampled
token rows of the named workloads and checks them against the oracle's exact
Y and dX with the parity bar max|got − exact| <= 1e-2·(|exact| + 1):

  - bf16 partials, each rounded by its rank (b added on rank 0) and summed
    with one bf16 rounding per ring step, as a 16-bit all-reduce does;
  - fp32 partials summed in rank order, plus b, rounded once to bf16, which
    is what the library's cross-GPU entry points do.

The emulated GPU arithmetic is the library's: Z in fp32, H and dH as bf16
(hi, lo) pairs (the accurate mode), fp32 accumulation of each partial.  It
calls no GPU code; it pins the choice of fp32 partials, not the kernels.
"""
import functools

import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import inputs


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _worst(got, exact):
    return float(np.max(np.abs(got - exact) / (1e-2 * (np.abs(exact) + 1.0))))


@functools.lru_cache(maxsize=1)
def _rows(name):
    """Exact Y, dX at 64 sampled rows and the library's per-rank partials'
    ingredients there (fp32 Z, the H and dH pairs)."""
    wl = inputs.WORKLOADS[name]
    inp = inputs.make_inputs(wl)
    rows = np.sort(np.random.default_rng(5).choice(wl.T, 64, replace=False))
    ex = oracle.sample_rows(inp, rows)
    X, dY = oracle.f64(inp["X"][rows]), oracle.f64(inp["dY"][rows])
    A, a, B, b = (oracle.f64(inp[k]) for k in ("A", "a", "B", "b"))
    Z32 = _f32(X @ A + a)
    H32 = _f32(oracle.gelu(Z32))
    dH32 = _f32(_f32(dY @ B.T) * oracle.gelu_grad(Z32))
    Hp = _bf16(H32) + _bf16(H32 - _bf16(H32))
    dHp = _bf16(dH32) + _bf16(dH32 - _bf16(dH32))
    return wl, ex, A, B, b, Hp, dHp


def _reduce(name, N):
    wl, ex, A, B, b, Hp, dHp = _rows(name)
    fs = wl.f // N
    P = [_f32(Hp[:, r * fs:(r + 1) * fs] @ B[r * fs:(r + 1) * fs]) for r in range(N)]
    Q = [_f32(dHp[:, r * fs:(r + 1) * fs] @ A[:, r * fs:(r + 1) * fs].T) for r in range(N)]
    # 16-bit all-reduce of each rank's rounded output
    y16, x16 = _bf16(P[0] + b), _bf16(Q[0])
    for r in range(1, N):
        y16, x16 = _bf16(y16 + _bf16(P[r])), _bf16(x16 + _bf16(Q[r]))
    # fp32 partials in rank order, b once, one rounding
    y32, x32 = P[0], Q[0]
    for r in range(1, N):
        y32, x32 = _f32(y32 + P[r]), _f32(x32 + Q[r])
    y32, x32 = _bf16(_f32(y32 + b)), _bf16(x32)
    return {"Y bf16": _worst(y16, ex["Y"]), "dX bf16": _worst(x16, ex["dX"]),
            "Y fp32": _worst(y32, ex["Y"]), "dX fp32": _worst(x32, ex["dX"])}


CASES = [(name, N) for name in ("tiny", "gpt2-medium", "h4096", "8.3b-class", "175b-class") for N in (2, 4, 8)]


@pytest.mark.parametrize("name,N", CASES, ids=[f"{n}-N{k}" for n, k in CASES])
def test_fp32_partials_meet_the_bar(name, N):
    r = _reduce(name, N)
    assert r["Y fp32"] < 0.75 and r["dX fp32"] < 0.75, r


@pytest.mark.parametrize("N", [2, 4, 8])
def test_bf16_partials_miss_the_bar_at_the_8p3b_class_workload(N):
    r = _reduce("8.3b-class", N)
    assert r["Y bf16"] > 1.2 and r["dX bf16"] > 1.2, r


def test_bf16_partials_miss_the_bar_at_the_175b_class_workload_on_8_ranks():
    r = _reduce("175b-class", 8)
    assert r["Y bf16"] > 1.0 and r["dX bf16"] > 1.0, r
