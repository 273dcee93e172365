"""Pins of the fp64 oracle against things other than itself (CPU only)."""
import math
import types

import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tests import oracle_pins as pins
from tensor_transformer_mlp_bias_b200 import inputs


# ------------------------------------------------------------------ GeLU
def test_gelu_fixed_points():
    assert oracle.gelu(np.array(0.0)) == 0.0
    assert oracle.gelu_grad(np.array(0.0)) == 0.5


def test_gelu_odd_part_is_identity():
    # g(x) - g(-x) = x·½(1+tanh u) + x·½(1-tanh u) = x, since tanh is odd.
    x = np.linspace(-9, 9, 3601)
    assert np.max(np.abs(oracle.gelu(x) - oracle.gelu(-x) - x)) < 1e-14


def test_gelu_asymptotes():
    x = np.array([8.0, 12.0, 30.0])
    assert np.allclose(oracle.gelu(x) / x, 1.0, rtol=0, atol=1e-14)
    assert np.all(np.abs(oracle.gelu(-x)) < 1e-14)
    assert np.allclose(oracle.gelu_grad(x), 1.0, atol=1e-12)
    assert np.all(np.abs(oracle.gelu_grad(-x)) < 1e-12)


def test_gelu_is_the_tanh_approximation_of_x_phi():
    # GELU(x) = x·Φ(x); the tanh form approximates it to < 5e-4 everywhere
    # and differs from it by more than 1e-4 somewhere (so it is not erf GELU).
    x = np.linspace(-10, 10, 20001)
    exact = 0.5 * x * (1 + np.vectorize(math.erf)(x / math.sqrt(2)))
    dev = np.abs(oracle.gelu(x) - exact)
    assert dev.max() < 5e-4
    assert dev.max() > 1e-4


def test_gelu_matches_torch_tanh_gelu():
    assert pins.pin_gelu_library(oracle) < 1e-14


def test_gelu_grad_central_difference():
    assert pins.pin_gelu_grad_fd(oracle) < 1e-8


# ------------------------------------------------------------------ the block
@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 4, 6), (5, 2, 8), (2, 6, 3)])
def test_brute_force_loops(shape):
    T, h, f = shape
    assert pins.pin_brute_force(oracle, pins.tiny_problem(T, h, f)) < 1e-12


@pytest.mark.parametrize("shape", [(3, 4, 6), (16, 32, 64), (7, 24, 40)])
def test_torch_float64_autograd(shape):
    T, h, f = shape
    assert pins.pin_autograd(oracle, pins.tiny_problem(T, h, f, seed=3)) < 1e-12


def test_finite_difference_gradients():
    assert pins.pin_finite_difference(oracle, pins.tiny_problem(4, 6, 10, seed=5)) < 1e-6


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_partition_invariant(t):
    p = pins.tiny_problem(9, 16, 64, seed=7)
    assert pins.pin_partition(oracle, p, t) < 1e-12


def test_shard_partials_are_the_column_row_blocks():
    # P_i must equal GeLU(X A_i + a_i) B_i computed directly from the blocks.
    p = pins.tiny_problem(5, 8, 12, seed=9)
    sf = oracle.forward_sharded(p["X"], p["A"], p["a"], p["B"], p["b"], 3)
    for i, P_i in enumerate(sf["partials"]):
        sl = slice(4 * i, 4 * i + 4)
        sub = oracle.forward(p["X"], p["A"][:, sl], p["a"][sl], p["B"][sl, :], np.zeros(8))
        assert pins.rel_err(P_i, sub["Y"]) < 1e-14
    # bias b enters once: t copies of b would shift Y by (t-1)·b
    assert pins.rel_err(sf["Y"], oracle.forward(p["X"], p["A"], p["a"], p["B"], p["b"])["Y"]) < 1e-14


def test_t1_is_a_plain_two_layer_mlp():
    p = pins.tiny_problem(6, 8, 16, seed=11)
    sf = oracle.forward_sharded(p["X"], p["A"], p["a"], p["B"], p["b"], 1)
    lin1 = torch.nn.Linear(8, 16).double()
    lin2 = torch.nn.Linear(16, 8).double()
    with torch.no_grad():
        lin1.weight.copy_(torch.tensor(p["A"].T))
        lin1.bias.copy_(torch.tensor(p["a"]))
        lin2.weight.copy_(torch.tensor(p["B"].T))
        lin2.bias.copy_(torch.tensor(p["b"]))
        y = lin2(torch.nn.functional.gelu(lin1(torch.tensor(p["X"])), approximate="tanh")).numpy()
    assert pins.rel_err(sf["Y"], y) < 1e-14


def test_shard_count_must_divide_ffn():
    with pytest.raises(ValueError):
        oracle.shard_slices(10, 4)


def test_sampled_values_equal_full_pass():
    wl = inputs.WORKLOADS["tiny"]
    inp = inputs.make_inputs(wl)
    ref = oracle.full(inp)
    rows = [0, 5, 63]
    cols = [0, 17, 511, 1023]
    sr = oracle.sample_rows(inp, rows)
    sc = oracle.sample_ffn(inp, cols)
    for k in ("Y", "Z", "H", "dX"):
        assert pins.rel_err(sr[k], ref[k][rows]) < 1e-13
    assert pins.rel_err(sc["dA"], ref["dA"][:, cols]) < 1e-13
    assert pins.rel_err(sc["da"], ref["da"][cols]) < 1e-13
    assert pins.rel_err(sc["dB"], ref["dB"][cols, :]) < 1e-13
    assert pins.rel_err(sc["db"], ref["db"]) < 1e-13


def test_flops_count():
    # six GEMMs of 2·T·h·f each; the tiny block is 2.01e8
    assert oracle.flops(64, 256, 1024) == 201326592


# ------------------------------------------------------------------ planted mistakes
def _mutant(**overrides):
    """A copy of the oracle module with some functions replaced."""
    m = types.SimpleNamespace(**{k: getattr(oracle, k) for k in dir(oracle) if not k.startswith("__")})
    for k, v in overrides.items():
        setattr(m, k, v)
    return m


def _fwd_bias_dropped(X, A, a, B, b):
    return oracle.forward(X, A, np.zeros_like(np.asarray(a, dtype=float)), B, b)


def _bwd_transposed_dA(dY, X, A, a, B):
    out = oracle.backward(dY, X, A, a, B)
    out["dA"] = out["dA"].T.copy() if out["dA"].shape[0] == out["dA"].shape[1] else out["dA"][::-1].copy()
    return out


def _gelu_grad_missing_term(x):
    u = oracle.SQRT_2_OVER_PI * (x + oracle.GELU_CUBIC * x ** 3)
    return 0.5 * (1.0 + np.tanh(u))


def _gelu_wrong_constant(x):
    u = oracle.SQRT_2_OVER_PI * (x + 0.0447 * x ** 3)
    return 0.5 * x * (1.0 + np.tanh(u))


def _fwd_sharded_bias_per_shard(X, A, a, B, b, t):
    out = oracle.forward_sharded(X, A, a, B, b, t)
    out["Y"] = out["Y"] + (t - 1) * np.asarray(b, dtype=float)[None, :]
    return out


def _bwd_sharded_gathered_dx(dY, X, A, a, B, t):
    out = oracle.backward_sharded(dY, X, A, a, B, t)
    out["dX"] = out["dX_partials"][0]  # keeps one shard instead of summing
    return out


@pytest.mark.parametrize("mutant,pin", [
    (_mutant(forward=_fwd_bias_dropped), "brute"),
    (_mutant(backward=_bwd_transposed_dA), "brute"),
    (_mutant(backward=_bwd_transposed_dA), "autograd"),
    (_mutant(gelu_grad=_gelu_grad_missing_term), "gelu_grad"),
    (_mutant(gelu=_gelu_wrong_constant), "gelu_lib"),
    (_mutant(forward_sharded=_fwd_sharded_bias_per_shard), "partition"),
    (_mutant(backward_sharded=_bwd_sharded_gathered_dx), "partition"),
])
def test_planted_mistake_is_caught(mutant, pin):
    p = pins.tiny_problem(4, 6, 6, seed=13)
    if pin == "brute":
        assert pins.pin_brute_force(mutant, p) > 1e-3
    elif pin == "autograd":
        assert pins.pin_autograd(mutant, p) > 1e-3
    elif pin == "gelu_grad":
        assert pins.pin_gelu_grad_fd(mutant) > 1e-3
    elif pin == "gelu_lib":
        assert pins.pin_gelu_library(mutant) > 1e-6
    elif pin == "partition":
        assert pins.pin_partition(mutant, p, 3) > 1e-3


def test_planted_mistake_in_backward_through_gelu_grad_is_caught():
    # backward() resolves gelu_grad from the module; plant it there.
    orig = oracle.gelu_grad
    try:
        oracle.gelu_grad = _gelu_grad_missing_term
        assert pins.pin_finite_difference(oracle, pins.tiny_problem(4, 6, 10, seed=5)) > 1e-3
    finally:
        oracle.gelu_grad = orig
