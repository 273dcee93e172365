"""Cross-GPU orchestration of the block (tensor_transformer_mlp_bias_b200.tp)
as two and four gloo ranks on the CPU.

Each rank holds one shard (its column block of A and a, its row block of B)
and runs the stage calls through the fp64 stand-in in tests/tp_cpu_ops.py;
the collectives are torch.distributed's.  Every rank checks its results
against the oracle's unsharded block: Y and dX (all-reduced, or its token
rows in the sequence-parallel form), its shard of dA, da and dB, and db.
This pins the host logic of the NCCL form (fp32 partials summed by the
collective, b added once after the sum, which outputs are reduced, gathered
or scattered, the shard and token bounds) and, with a stand-in for CUDA IPC,
the peer-table exchange of the fused form.  The GEMMs and the fused
reduction are checked on the GPU elsewhere; runs on several GPUs are not
possible on a one-GPU machine.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tensor_transformer_mlp_bias_b200 import tp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, shape, sp, mode, results):
    import torch.distributed as dist
    from oracle import mlp_oracle as oracle
    from tensor_transformer_mlp_bias_b200 import inputs
    from tests import tp_cpu_ops
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, h, f = shape
        inp = inputs.make_custom(T, h, f, seed=11)
        ref = oracle.full(inp)
        d = {k: v.to(torch.float64) for k, v in inp.items()}
        A_i, a_i, B_i = tp.shard_parameters(d["A"], d["a"], d["B"], rank, world)
        lo, hi = tp.shard_bounds(f, rank, world)
        rows = tp.token_rows(T, rank, world) if sp else slice(0, T)
        X = d["X"][rows] if sp else d["X"]
        dY = d["dY"][rows] if sp else d["dY"]
        Y, saved = tp.forward(X, A_i, a_i, B_i, d["b"], sequence_parallel=sp, mode=mode, reduction="nccl", ops=tp_cpu_ops)
        g = tp.backward(dY, saved, A_i, B_i, sequence_parallel=sp, mode=mode, reduction="nccl", ops=tp_cpu_ops)
        err = {
            "Y": np.abs(Y.numpy() - ref["Y"][rows]).max(),
            "dX": np.abs(g["dX"].numpy() - ref["dX"][rows]).max(),
            "dA": np.abs(g["dA"].numpy() - ref["dA"][:, lo:hi]).max(),
            "da": np.abs(g["da"].numpy() - ref["da"][lo:hi]).max(),
            "dB": np.abs(g["dB"].numpy() - ref["dB"][lo:hi, :]).max(),
            "db": np.abs(g["db"].numpy() - ref["db"]).max(),
        }
        scale = {k: 1.0 + float(np.abs(ref[k]).max()) for k in err}
        results[rank] = {k: float(v) / scale[k] for k, v in err.items()}
    finally:
        dist.destroy_process_group()


def _run(world, shape, sp, mode):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, sp, mode, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    return dict(results)


@pytest.mark.parametrize("sp", [False, True], ids=["tensor_parallel", "sequence_parallel"])
@pytest.mark.parametrize("mode", [0, 3, 4], ids=["accurate", "fast", "fp8"])
def test_two_ranks_match_the_unsharded_block(sp, mode):
    res = _run(2, (64, 128, 256), sp, mode)
    assert set(res) == {0, 1}
    for rank, errs in res.items():
        for k, e in errs.items():
            assert e < 1e-12, (rank, k, e)


@pytest.mark.parametrize("mode", [0, 4], ids=["accurate", "fp8"])
def test_four_ranks_sequence_parallel_match_the_unsharded_block(mode):
    res = _run(4, (64, 128, 512), True, mode)
    assert set(res) == {0, 1, 2, 3}
    for rank, errs in res.items():
        for k, e in errs.items():
            assert e < 1e-12, (rank, k, e)


def test_shard_and_token_bounds():
    assert tp.shard_bounds(1024, 0, 4) == (0, 256)
    assert tp.shard_bounds(1024, 3, 4) == (768, 1024)
    assert tp.token_rows(64, 1, 2) == slice(32, 64)
    with pytest.raises(ValueError):
        tp.shard_bounds(1000, 0, 3)
    with pytest.raises(ValueError):
        tp.token_rows(63, 0, 2)
    A = torch.arange(4 * 8, dtype=torch.float64).view(4, 8)
    a = torch.arange(8, dtype=torch.float64)
    B = torch.arange(8 * 4, dtype=torch.float64).view(8, 4)
    A1, a1, B1 = tp.shard_parameters(A, a, B, 1, 2)
    assert torch.equal(A1, A[:, 4:]) and torch.equal(a1, a[4:]) and torch.equal(B1, B[4:, :])
    assert A1.is_contiguous() and B1.is_contiguous()


# ------------------------------------------------------------------ peer table of the fused form
class _FakeIpc:
    """Stand-in for the library's CUDA IPC calls: an address exported by rank
    r maps, in rank q's process, to 1e12·(q+1) + address (a fake mapping)."""
    def __init__(self, rank):
        self.rank = rank
        self.closed = []

    def mlp_tp_ipc_export(self, ptr):
        return (f"handle-of-rank-{self.rank}".encode(), ptr % 4096)

    def mlp_tp_ipc_import(self, handle, offset):
        src = int(handle.decode().rsplit("-", 1)[1])
        return (self.rank + 1) * 10 ** 12 + src * 10 ** 9 + offset

    def mlp_tp_ipc_close(self, ptr, offset):
        self.closed.append((ptr, offset))

    def peer_recv_bytes(self, T, h, world):
        return T * h * 4

    def peer_flag_bytes(self, T, h, world):
        return 256

    def make_peer(self, rank, world, recv, flags=None, epoch=0):
        return {"rank": rank, "world": world, "recv": list(recv), "flags": list(flags), "epoch": epoch}


def _exchange_worker(rank, world, port, results):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ipc = _FakeIpc(rank)
        ex = tp.PeerExchange(64 * world, 128, device="cpu", ops=ipc)
        own = ex.buf.data_ptr()
        q1, q2 = ex.next(), ex.next()
        ex.close()
        results[rank] = {"own": own, "table": ex.table, "q1": q1, "q2": q2, "closed": ipc.closed,
                         "recv_bytes": ex.recv_bytes}
    finally:
        dist.destroy_process_group()


def test_peer_exchange_maps_every_other_rank_and_keeps_its_own_pointer():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for rank in range(world):
        res = results[rank]
        table = res["table"]
        assert len(table) == world and table[rank] == res["own"]
        for src in range(world):
            if src != rank:
                # the mapping of rank src's exported buffer, at its offset inside its allocation
                off = results[src]["own"] % 4096
                assert table[src] == (rank + 1) * 10 ** 12 + src * 10 ** 9 + off
        q1, q2 = res["q1"], res["q2"]
        assert (q1["rank"], q1["world"], q1["epoch"], q2["epoch"]) == (rank, world, 1, 2)
        assert q1["recv"] == table and q1["flags"] == [a + res["recv_bytes"] for a in table]
        assert sorted(res["closed"]) == sorted((table[s], results[s]["own"] % 4096) for s in range(world) if s != rank)
