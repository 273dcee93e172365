"""The cross-GPU orchestration (tensor_transformer_mlp_bias_b200.tp) on the
GPU through the C-ABI, as one NCCL rank in a child process.

With one rank the collectives move nothing, but every stage runs through the
library with the shard shapes the orchestration passes (t = 1 per rank), in
both reduction forms (the fused peer-store reduction and the NCCL one over
fp32 partials), and the results must meet the parity bar against the
oracle's unsharded block.
Several ranks need several GPUs; this machine gives one.
"""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(port, sp, mode, reduction, results):
    import torch
    import torch.distributed as dist
    from oracle import mlp_oracle as oracle
    from tensor_transformer_mlp_bias_b200 import inputs, tp
    from tests.parity_util import worst_ratio
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        T, h, f = 384, 256, 1024
        inp = inputs.make_custom(T, h, f, seed=21)
        ref = oracle.full(inp)
        d = {k: v.cuda() for k, v in inp.items()}
        A_i, a_i, B_i = tp.shard_parameters(d["A"], d["a"], d["B"], 0, 1)
        Y, saved = tp.forward(d["X"], A_i, a_i, B_i, d["b"], sequence_parallel=sp, mode=mode, reduction=reduction)
        g = tp.backward(d["dY"], saved, A_i, B_i, sequence_parallel=sp, mode=mode, reduction=reduction)
        torch.cuda.synchronize()
        out = dict(g, Y=Y)
        results["ratios"] = {k: worst_ratio(out[k], ref[k]) for k in ("Y", "dX", "dA", "da", "dB", "db")}
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("sp", [False, True], ids=["tensor_parallel", "sequence_parallel"])
@pytest.mark.parametrize("mode", [0, 3, 4], ids=["accurate", "fast", "fp8"])
@pytest.mark.parametrize("reduction", ["peer", "nccl"])
def test_one_rank_through_the_library_meets_the_bar(sp, mode, reduction):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    p = ctx.Process(target=_worker, args=(_free_port(), sp, mode, reduction, results))
    p.start()
    p.join(300)
    assert p.exitcode == 0
    for k, w in results["ratios"].items():
        assert w <= 1.0, (k, w)
