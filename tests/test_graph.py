"""The composite calls inside a CUDA graph.

The C-ABI enqueues only kernel launches, asynchronous memsets and (in the fp8
mode) an event fork and join with its own side stream on the
caller's stream.  It allocates nothing and does not synchronise, so a whole
forward+backward can be captured once and replayed, which removes the host's
launch cost for small batches.  A replay must give the same bits as eager
execution, also after new input values are copied into the captured buffers.
"""
import pytest
import torch

from tensor_transformer_mlp_bias_b200 import binding, block, inputs
from tests.parity_util import bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,mode", [((64, 256, 1024, 2), binding.FAST),
                                        ((333, 320, 1280, 5), binding.ACCURATE),
                                        ((333, 320, 1280, 5), binding.FP8)],
                         ids=["tiny_fast", "ragged_accurate", "ragged_fp8"])
def test_graph_replay_matches_eager(shape, mode):
    T, h, f, t = shape
    inp = {k: v.cuda() for k, v in inputs.make_custom(T, h, f, seed=51).items()}
    out = block.alloc_outputs(T, h, f, mode=mode)
    ws = binding.make_workspace_mode(T, h, f, t, mode)  # the fp8 mode forks its operand copies onto a side stream

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm up (kernel attributes, occupancy) outside the capture
        block.forward(inp, t, out, ws, mode)
        block.backward(inp, t, out, ws, mode)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        block.forward(inp, t, out, ws, mode)
        block.backward(inp, t, out, ws, mode)

    for seed in (52, 53):
        fresh = inputs.make_custom(T, h, f, seed=seed)
        for k, v in fresh.items():
            inp[k].copy_(v)
        g.replay()
        torch.cuda.synchronize()
        binding.mlp_tp_check(ws)
        eager = block.forward_backward({k: v.clone() for k, v in inp.items()}, t, mode=mode)
        for k in ("Y", "Z", "H", "H_lo", "dX", "dA", "da", "dB", "db"):
            a, b = out[k], eager[k]
            same = torch.equal(a.view(torch.uint8), b.view(torch.uint8))
            assert same, (seed, k)
