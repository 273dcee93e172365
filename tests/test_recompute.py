"""Activation recomputation: the forward keeps Z, H, H_lo only in the
workspace and the backward recomputes them from X.  The recomputed
activations come from the same kernels, so every output must equal the
saved-activation path bit for bit, and the oracle within the parity bar."""
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import binding, block, inputs
from tests.parity_util import assert_close, bits

pytestmark = pytest.mark.gpu


def _recompute(inp, t, mode):
    T, h = inp["X"].shape
    f = inp["A"].shape[1]
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    out = {"Y": e(T, h), "dX": e(T, h), "dA": e(h, f), "da": e(f), "dB": e(f, h), "db": e(h)}
    ws = binding.make_recompute_workspace(T, h, f, t)
    binding.mlp_tp_forward_recompute(inp["X"], inp["A"], inp["a"], inp["B"], inp["b"], T, h, f, t, mode,
                                     out["Y"], ws)
    # anything may reuse the workspace between forward and backward
    ws[:].fill_(0)
    binding.mlp_tp_backward_recompute(inp["dY"], inp["X"], inp["A"], inp["a"], inp["B"], T, h, f, t, mode,
                                      out["dX"], out["dA"], out["da"], out["dB"], out["db"], ws)
    binding.mlp_tp_check(ws)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("shape,mode", [((200, 192, 384, 6), binding.ACCURATE), ((333, 320, 1280, 5), binding.FAST),
                                        ((64, 256, 1024, 2), binding.ACCURATE)])
def test_recompute_matches_saved_path_and_oracle(shape, mode):
    T, h, f, t = shape
    host = inputs.make_custom(T, h, f, seed=31 + T)
    inp = {k: v.cuda() for k, v in host.items()}
    rec = _recompute(inp, t, mode)
    saved = block.forward_backward(inp, t, mode=mode)
    torch.cuda.synchronize()
    for k in rec:
        assert torch.equal(bits(rec[k]), bits(saved[k])), k
    ref = oracle.full(host)
    for k in rec:
        assert_close(k, rec[k], ref[k])


def test_recompute_bitwise_at_h4096():
    wl = inputs.WORKLOADS["h4096"]
    inp = {k: v.cuda() for k, v in inputs.make_inputs(wl).items()}
    rec = _recompute(inp, 8, binding.ACCURATE)
    saved = block.forward_backward(inp, 8)
    torch.cuda.synchronize()
    for k in rec:
        assert torch.equal(bits(rec[k]), bits(saved[k])), k
