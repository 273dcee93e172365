"""Failure detection without a GPU fault.

Every wait inside the GEMM kernels is bounded.  A test hook makes the
operand-loading warp stop after one pipeline stage, so the tensor-core warp
waits for a stage that never arrives; the wait runs out of its budget, the
kernel records MLP_ERR_TIMEOUT in the workspace status word, drains its own
in-flight copies and MMAs, frees its TMEM and returns.  The host reads the
status with mlp_tp_check, and the next, normal call on the same context must
succeed and be correct.
"""
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import binding, inputs
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu


def _fc1(inp, T, h, f, t, ws):
    Z = torch.empty(T, f, dtype=torch.float32, device="cuda")
    H = torch.empty(T, f, dtype=torch.bfloat16, device="cuda")
    H_lo = torch.empty_like(H)
    binding.mlp_tp_fc1_forward(inp["X"], inp["A"], inp["a"], T, h, f, t, Z, H, H_lo, ws)
    return Z, H


def test_bounded_wait_reports_timeout_and_context_survives():
    T, h, f, t = 512, 512, 2048, 2
    host = inputs.make_custom(T, h, f, seed=21)
    inp = {k: v.cuda() for k, v in host.items()}
    ws = binding.make_workspace(T, h, f, t)
    try:
        binding.mlp_tp_set_wait_budget_ns(20_000_000)  # 20 ms per wait
        binding.mlp_tp_set_debug_flags(1)
        _fc1(inp, T, h, f, t, ws)
        with pytest.raises(binding.MlpError) as e:
            binding.mlp_tp_check(ws)
        assert e.value.status == 7, str(e.value)  # MLP_ERR_TIMEOUT
    finally:
        binding.mlp_tp_set_debug_flags(0)
        binding.mlp_tp_set_wait_budget_ns(1_000_000_000)
    # the status word was cleared by the check; the context is usable
    Z, H = _fc1(inp, T, h, f, t, ws)
    binding.mlp_tp_check(ws)
    ref = oracle.forward(host["X"], host["A"], host["a"], host["B"], host["b"])
    assert_close("Z after timeout", Z, ref["Z"])
    assert_close("H after timeout", H, ref["H"])
