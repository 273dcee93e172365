"""The bounds-checking build (-DMLPTP_BOUNDS_CHECK) on the GPU.

In that build every plain global access that does not go through a tensor
map (the column-sum partials, the fp32 pieces of split tiles and their
reduce, the bias-gradient column sums) checks its index against its buffer
and reports MLP_ERR_BOUNDS from mlp_tp_check instead of touching memory
outside it.  It stands in for a memory checker, which this machine does not
offer.  The shapes below reach every checked site: split shard-sum tails,
K-split weight gradients, ragged tiles, da and db, a batch whose [T, f]
tensors hold more than 2^31 elements, the allocation-free path, and the
cross-GPU path's peer stores and reduce (two ranks emulated on this GPU), and
the fp16 + e4m3 mode.  They must pass with a clean status
word and meet the parity bar.
"""
import os
import subprocess
import sys

import pytest

from tensor_transformer_mlp_bias_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1])
from tensor_transformer_mlp_bias_b200 import binding
binding.LIB_PATH = sys.argv[2]
from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import block, inputs
from tests.parity_util import assert_close, to_gpu
shapes = [(333, 320, 1280, 5, 3), (1024, 256, 1024, 2, 3), (2048, 128, 512, 4, 0), (1, 64, 128, 2, 3),
          (257, 512, 768, 3, 0),
          # the fp16 + e4m3 mode: casts, statistics, the e4m3 stages' ragged token tail, K-split pieces
          (333, 320, 1280, 5, 4), (1024, 256, 1024, 2, 4), (129, 192, 768, 3, 4)]
for T, h, f, t, mode in shapes:
    inp = inputs.make_custom(T, h, f, seed=T + f)
    out = block.forward_backward(to_gpu(inp), t, mode=mode)  # mlp_tp_check raises on MLP_ERR_BOUNDS
    ref = oracle.full(inp)
    for k in ("Y", "dX", "dA", "da", "dB", "db"):
        assert_close(k, out[k], ref[k])
import numpy as np
import torch
# T*f above 2^31 elements: every plain index must be 64-bit (sampled oracle)
T, h, f, t = 65536, 1024, 33280, 8
inp = inputs.make_custom(T, h, f, seed=71)
out = block.forward_backward(to_gpu(inp), t)
rows = np.array([0, 1, 30000, 65535])
cols = np.array([0, 5, 20000, 33279])
sr = oracle.sample_rows(inp, rows)
sc = oracle.sample_ffn(inp, cols)
r = torch.as_tensor(rows, device="cuda")
c = torch.as_tensor(cols, device="cuda")
assert_close("Y rows", out["Y"][r], sr["Y"])
assert_close("dX rows", out["dX"][r], sr["dX"])
assert_close("dA cols", out["dA"][:, c], sc["dA"])
assert_close("dB rows", out["dB"][c, :], sc["dB"])
assert_close("da cols", out["da"][c], sc["da"])
del out
torch.cuda.empty_cache()
# the same batch in the fp16 + e4m3 mode (e4m3 [T, f] tensors of 2.18e9 bytes)
out = block.forward_backward(to_gpu(inp), t, mode=binding.FP8)
assert_close("Y rows (fp8)", out["Y"][r], sr["Y"])
assert_close("dX rows (fp8)", out["dX"][r], sr["dX"])
assert_close("dA cols (fp8)", out["dA"][:, c], sc["dA"])
assert_close("dB rows (fp8)", out["dB"][c, :], sc["dB"])
del out, inp
torch.cuda.empty_cache()
T, h = 4096, 1024
dY = to_gpu(inputs.make_custom(T, h, 256, seed=3))["dY"]
db = torch.empty(h, dtype=torch.bfloat16, device="cuda")  # h elements, as the call writes
binding.mlp_tp_fc2_bias_grad_noalloc(dY, T, h, db)
binding.mlp_tp_check(None)  # the allocation-free path's own status word: raises on MLP_ERR_BOUNDS
assert_close("db (allocation-free)", db, dY.double().sum(0).cpu().numpy())
# the cross-GPU path: peer stores from the GEMM epilogue and the owner's reduce, two ranks emulated in stream
# order on this GPU (no wait spins), forward and backward partials on the same buffers
from tensor_transformer_mlp_bias_b200 import tp
T, h, f, N = 512, 384, 1024, 2
host = inputs.make_custom(T, h, f, seed=81)
inp = to_gpu(host)
ref = oracle.full(host)
fs = f // N
rb, fb = binding.peer_recv_bytes(T, h, N), binding.peer_flag_bytes(T, h, N)
recv = [torch.zeros(rb, dtype=torch.uint8, device="cuda") for _ in range(N)]
flags = [torch.zeros(fb, dtype=torch.uint8, device="cuda") for _ in range(N)]
acts = []
for r in range(N):
    A_i, a_i, B_i = tp.shard_parameters(inp["A"], inp["a"], inp["B"], r, N)
    ws = binding.make_workspace(T, h, fs, 1)
    Z = torch.empty(T, fs, dtype=torch.float32, device="cuda")
    H, H_lo, dH, dH_lo = (torch.empty(T, fs, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    binding.mlp_tp_fc1_forward(inp["X"], A_i, a_i, T, h, fs, 1, Z, H, H_lo, ws)
    binding.mlp_tp_fc2_backward_data(inp["dY"], B_i, Z, T, h, fs, 1, dH, dH_lo, None, ws)
    acts.append((A_i, B_i, H, H_lo, dH, dH_lo, ws))
for epoch, what in ((1, "Y"), (2, "dX")):
    qs = [binding.make_peer(r, N, recv, flags, epoch) for r in range(N)]
    for r, (A_i, B_i, H, H_lo, dH, dH_lo, ws) in enumerate(acts):
        if what == "Y":
            binding.mlp_tp_fc2_forward_peer(H, H_lo, B_i, T, h, fs, qs[r], ws)
        else:
            binding.mlp_tp_fc1_backward_data_peer(dH, dH_lo, A_i, T, h, fs, qs[r], ws)
    outs = []
    for o in range(N):
        out = torch.empty(T // N, h, dtype=torch.bfloat16, device="cuda")
        binding.mlp_tp_peer_reduce(qs[o], inp["b"] if what == "Y" else None, T, h, out, acts[o][6])
        outs.append(out)
    for a in acts:
        binding.mlp_tp_check(a[6])  # raises on MLP_ERR_BOUNDS
    assert_close(what + " (cross-GPU path)", torch.cat(outs), ref[what])
print("bounds-checked build: clean")
"""


def test_bounds_checked_build_is_clean(tmp_path):
    lib = build.build(defines=["MLPTP_BOUNDS_CHECK"], out=str(tmp_path / "libmlptp_bounds.so"))
    res = subprocess.run([sys.executable, "-c", CHILD, ROOT, lib], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    assert "clean" in res.stdout
