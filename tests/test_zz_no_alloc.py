"""The allocation-free bias-gradient entry point.

Some callers cannot hand the library a workspace: a serving process whose
memory pool already owns all of HBM, or a plugin interface that passes only
input and output pointers.  mlp_tp_fc2_bias_grad_noalloc computes
db = Σ_rows dY for them with its scratch in a static device array inside the
library.  These tests call it through the C-ABI and check it against the
workspace entry point mlp_tp_fc2_backward_weight, twice in a row (the array
keeps the previous call's contents, which must not leak into the next
result), and check that too-large shapes are refused.

This file is named to be collected last.
"""
import pytest
import torch

from tensor_transformer_mlp_bias_b200 import binding, inputs
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu


def _db_with_workspace(inp, t):
    T, h = inp["dY"].shape
    f = inp["B"].shape[0]
    ws = binding.make_workspace(T, h, f, t)
    H = torch.zeros(T, f, dtype=torch.bfloat16, device="cuda")
    dB = torch.empty(f, h, dtype=torch.bfloat16, device="cuda")
    db = torch.empty(h, dtype=torch.bfloat16, device="cuda")
    binding.mlp_tp_fc2_backward_weight(H, H, inp["dY"], T, h, f, t, dB, db, ws)
    binding.mlp_tp_check(ws)
    return db


def test_noalloc_bias_grad_matches_workspace_path_twice():
    shapes = [(4096, 1024, 4096, 4), (333, 512, 1024, 2)]  # the second call is smaller: stale data must not leak
    for T, h, f, t in shapes:
        inp = {k: v.cuda() for k, v in inputs.make_custom(T, h, f, seed=T).items()}
        ref = _db_with_workspace(inp, t)
        db = torch.full((h,), 99.0, dtype=torch.bfloat16, device="cuda")
        binding.mlp_tp_fc2_bias_grad_noalloc(inp["dY"], T, h, db)
        binding.mlp_tp_check(None)  # syncs; the path's own status word is clean
        assert_close("db (allocation-free)", db, ref.double().cpu().numpy())


def test_noalloc_bias_grad_refuses_shapes_beyond_its_scratch():
    h = 4096
    T = 257 * 256  # ceil(T/256)·h = 257·4096 > 2^20 partials
    dY = torch.empty(8, h, dtype=torch.bfloat16, device="cuda")  # never read: the call is refused first
    db = torch.empty(h, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.MlpError) as e:
        binding.mlp_tp_fc2_bias_grad_noalloc(dY, T, h, db)
    assert e.value.status == 2 and "allocation-free" in str(e.value)


def test_noalloc_bias_grad_empty_batch_gives_zeros():
    h = 256
    db = torch.full((h,), 5.0, dtype=torch.bfloat16, device="cuda")
    binding.mlp_tp_fc2_bias_grad_noalloc(None, 0, h, db)
    torch.cuda.synchronize()
    assert bool((db == 0).all())
