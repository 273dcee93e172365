"""The precision of the saved intermediates, checked on the CPU.

The pages keep the activations of the block in bf16 or fp16 and say nothing
finer about the pre-activation Z, the activation H = g(Z) or the activation
gradient dH.  Against the exact fp64 block and the bar
max|gpu - exact| <= 1e-2·(|exact| + 1), the library keeps Z in fp32 and H, dH
as bf16 (hi, lo) pairs, and forms the weight gradients dA = Xᵀ·dH and
dB = Hᵀ·dY over both halves.  This test emulates the candidate roundings in
fp64 at sampled ffn columns of the GPT-2-medium workload (T=8192, h=1024,
f=4096; exact values from the oracle) and checks which side of the bar each
lands on:

  - H or dH rounded to bf16: dB or dA misses the bar by a wide margin;
  - the (hi, lo) pairs with Z in fp32: both inside it;
  - the dH pair formed from a bf16-rounded Z: dA still misses it.

It calls no GPU code; it pins the reading, not the kernels.
"""
import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import inputs


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _f32(x: np.ndarray) -> np.ndarray:
    return x.astype(np.float32).astype(np.float64)


def _pair(x: np.ndarray):
    hi = _bf16(x)
    return hi, _bf16(x - hi)


def _worst(got: np.ndarray, exact: np.ndarray) -> float:
    """Worst |got - exact| as a multiple of the parity tolerance."""
    return float(np.max(np.abs(got - exact) / (1e-2 * (np.abs(exact) + 1.0))))


@pytest.fixture(scope="module")
def sampled():
    wl = inputs.WORKLOADS["gpt2-medium"]
    inp = inputs.make_inputs(wl)
    cols = np.sort(np.random.default_rng(7).choice(wl.f, 16, replace=False))
    exact = oracle.sample_ffn(inp, cols)
    X, A, a, B, dY = (inp[k].double().numpy() for k in ("X", "A", "a", "B", "dY"))
    Z32 = _f32(X @ A[:, cols] + a[cols])  # fp32 accumulation of the GEMM, kept in fp32
    dG = _f32(dY @ B[cols].T)
    return {"exact": exact, "X": X, "dY": dY, "Z32": Z32, "dG": dG}


def test_bf16_activation_misses_the_bar_for_dB(sampled):
    H = _f32(oracle.gelu(sampled["Z32"]))
    dB = _bf16(_bf16(H).T @ sampled["dY"])
    assert _worst(dB, sampled["exact"]["dB"]) > 3.0


def test_activation_pair_meets_the_bar_for_dB(sampled):
    H = _f32(oracle.gelu(sampled["Z32"]))
    hi, lo = _pair(H)
    dB = _bf16((hi + lo).T @ sampled["dY"])
    assert _worst(dB, sampled["exact"]["dB"]) < 0.75


def test_bf16_gradient_misses_the_bar_for_dA(sampled):
    dH = _f32(sampled["dG"] * oracle.gelu_grad(sampled["Z32"]))
    dA = _bf16(sampled["X"].T @ _bf16(dH))
    assert _worst(dA, sampled["exact"]["dA"]) > 3.0


def test_gradient_pair_from_fp32_z_meets_the_bar_for_dA(sampled):
    dH = _f32(sampled["dG"] * oracle.gelu_grad(sampled["Z32"]))
    hi, lo = _pair(dH)
    dA = _bf16(sampled["X"].T @ (hi + lo))
    assert _worst(dA, sampled["exact"]["dA"]) < 0.75
    # da is summed from the fp32 dH
    assert _worst(_bf16(_f32(dH.sum(axis=0))), sampled["exact"]["da"]) < 0.75


def test_gradient_pair_from_bf16_z_misses_the_bar_for_dA(sampled):
    dH = _f32(sampled["dG"] * oracle.gelu_grad(_bf16(sampled["Z32"])))
    hi, lo = _pair(dH)
    dA = _bf16(sampled["X"].T @ (hi + lo))
    assert _worst(dA, sampled["exact"]["dA"]) > 3.0
