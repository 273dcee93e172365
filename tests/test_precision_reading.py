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


# ------------------------------------------------------------------ the fp16 + e4m3 mode
# The roundings of MLP_TP_FP8, emulated: fp16 high parts (11 bits) and e4m3
# residuals (4 bits) 2^7 apart, power-of-two scales from the same statistics
# the library reduces (max|X|, max|dY|, the largest row norms of dY and B).
def _f16(x):
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float64)


def _e4m3(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).double().numpy()


def _pow2_below(e_target, v):
    """Largest power of two s with v·s <= 2^e_target (v > 0)."""
    m, e = np.frexp(v)  # v = m·2^e, m in [0.5, 1)
    return 2.0 ** (e_target - (e - 1) - (0 if m == 0.5 else 1))


@pytest.fixture(scope="module")
def fp8_scales():
    wl = inputs.WORKLOADS["gpt2-medium"]
    inp = inputs.make_inputs(wl)
    X, B, dY = (inp[k].double().numpy() for k in ("X", "B", "dY"))
    sX = _pow2_below(15, np.abs(X).max())
    sY = _pow2_below(15, np.abs(dY).max())
    bound = 1.212 * np.sqrt((dY ** 2).sum(1).max()) * np.sqrt((B ** 2).sum(1).max())
    return {"sX": sX, "sY": sY, "sH": _pow2_below(12, bound), "inp": inp}


def test_fp8_scale_rule_keeps_the_residual_in_range(sampled, fp8_scales):
    """|dH·sH| < 2^13 (the e4m3 residual cannot saturate) and the fp16 and
    e4m3 copies of X and dY stay below 2^15 and 2^8."""
    dH = _f32(sampled["dG"] * oracle.gelu_grad(sampled["Z32"]))
    assert np.abs(dH).max() * fp8_scales["sH"] < 2.0 ** 13
    assert np.abs(sampled["X"]).max() * fp8_scales["sX"] <= 2.0 ** 15
    assert np.abs(sampled["dY"]).max() * fp8_scales["sY"] / 128.0 <= 2.0 ** 8


def test_fp16_e4m3_weight_gradients_meet_the_bar(sampled, fp8_scales):
    sX, sY, sH = fp8_scales["sX"], fp8_scales["sY"], fp8_scales["sH"]
    X, dY = sampled["X"], sampled["dY"]
    H = _f32(oracle.gelu(sampled["Z32"]))
    H16 = _f16(H)
    H8 = _e4m3((H - H16) * 128.0)
    dB = _bf16(_f32(_f32(H16.T @ _f16(dY * sY)) + _f32(H8.T @ _e4m3(dY * sY / 128.0))) / sY)
    assert _worst(dB, sampled["exact"]["dB"]) < 0.75
    ds = _f32(sampled["dG"] * oracle.gelu_grad(sampled["Z32"])) * sH
    dH16 = _f16(ds)
    dH8 = _e4m3((ds - dH16) * 128.0)
    dA = _bf16(_f32(_f32(_f16(X * sX).T @ dH16) + _f32(_e4m3(X * sX / 128.0).T @ dH8)) / (sX * sH))
    assert _worst(dA, sampled["exact"]["dA"]) < 0.75


def test_fp16_products_meet_the_bar_for_y_and_dx(fp8_scales):
    """Y = H16·fp16(B) + b and dX = dH16·fp16(A)ᵀ / sH at sampled rows."""
    inp = fp8_scales["inp"]
    X, A, a, B, b, dY = (inp[k].double().numpy() for k in ("X", "A", "a", "B", "b", "dY"))
    rows = np.sort(np.random.default_rng(5).choice(X.shape[0], 8, replace=False))
    exact = oracle.sample_rows(inp, rows)
    Z = _f32(X[rows] @ A + a)
    Y = _bf16(_f32(_f16(_f32(oracle.gelu(Z))) @ _f16(B)) + b)
    assert _worst(Y, exact["Y"]) < 0.75
    sH = fp8_scales["sH"]
    dH16 = _f16(_f32(_f32(dY[rows] @ B.T) * oracle.gelu_grad(Z)) * sH)
    dX = _bf16(_f32(dH16 @ _f16(A).T) / sH)
    assert _worst(dX, exact["dX"]) < 0.75
