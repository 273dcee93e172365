"""Parity at a batch whose [T, f] tensors hold more than 2^31 elements
(T = 65536, h = 1024, f = 33280, t = 8; about 28 GB on the device), through
the normal build: every index of the path is 64-bit where it must be.  The
bounds-checking build runs the same batch first (tests/test_bounds_build.py).
The oracle is evaluated exactly at sampled token rows and ffn indices."""
import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import block, inputs
from tests.parity_util import assert_close, to_gpu

pytestmark = pytest.mark.gpu


def test_more_than_2_31_elements_per_activation():
    T, h, f, t = 65536, 1024, 33280, 8
    assert T * f > 2 ** 31
    inp = inputs.make_custom(T, h, f, seed=71)
    out = block.forward_backward(to_gpu(inp), t)
    rows = np.array([0, 1, 2 ** 15 + 3, T - 1])
    cols = np.array([0, 7, 2 ** 14 + 5, f - 1])
    sr = oracle.sample_rows(inp, rows)
    sc = oracle.sample_ffn(inp, cols)
    r = torch.as_tensor(rows, device="cuda")
    c = torch.as_tensor(cols, device="cuda")
    assert_close("Y rows", out["Y"][r], sr["Y"])
    assert_close("Z rows", out["Z"][r], sr["Z"])
    assert_close("H rows", out["H"][r], sr["H"])
    assert_close("dX rows", out["dX"][r], sr["dX"])
    assert_close("dA cols", out["dA"][:, c], sc["dA"])
    assert_close("da cols", out["da"][c], sc["da"])
    assert_close("dB rows", out["dB"][c, :], sc["dB"])
    assert_close("db", out["db"], sc["db"])
    del out
    torch.cuda.empty_cache()
