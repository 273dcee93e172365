"""The fused cross-GPU shard reduction (mlp_tp_*_peer, mlp_tp_peer_reduce) on
one GPU.

Each rank's row-parallel GEMM stores its fp32 partial, block by block, into
the receive buffer of the rank that owns those token rows and raises the
block's arrival count; the owner's reduce kernel adds the partials in rank
order plus the bias and rounds once.  This machine gives one GPU, so:

  - one rank (world = 1) must reproduce the single-GPU stage calls with t = 1
    bit for bit, over several exchanges on the same buffers;
  - N ranks are emulated on the one GPU: every rank's GEMM, then every
    owner's reduce, launched one after another on one stream.  The peer table
    then holds N buffers of this GPU, so the kernels run the same routing,
    slots, counters and consumed marks as on N GPUs, and no wait ever spins
    (each kernel starts after the ones it waits for have finished);
  - the bounded waits are made to run out (a flag nobody sets) and must
    report MLP_ERR_TIMEOUT, with the context usable afterwards;
  - a second process maps a buffer of the first through the library's IPC
    calls and reads it with a reduce (epoch 0, nothing waits).

Several GPUs would be needed to run the ranks concurrently; that is not
possible here.
"""
import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import binding, inputs, tp
from tests.parity_util import assert_close, bits

pytestmark = pytest.mark.gpu


def _zeros_bytes(n):
    return torch.zeros(n, dtype=torch.uint8, device="cuda")


def _activations(inp, A_i, a_i, B_i, T, h, fs):
    """This rank's Z, H, H_lo and dH, dH_lo through the single-GPU stage calls (t = 1)."""
    ws = binding.make_workspace(T, h, fs, 1)
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    Z = torch.empty(T, fs, dtype=torch.float32, device="cuda")
    H, H_lo, dH, dH_lo = e(T, fs), e(T, fs), e(T, fs), e(T, fs)
    binding.mlp_tp_fc1_forward(inp["X"], A_i, a_i, T, h, fs, 1, Z, H, H_lo, ws)
    binding.mlp_tp_fc2_backward_data(inp["dY"], B_i, Z, T, h, fs, 1, dH, dH_lo, None, ws)
    binding.mlp_tp_check(ws)
    return {"H": H, "H_lo": H_lo, "dH": dH, "dH_lo": dH_lo, "ws": ws}


@pytest.mark.parametrize("T,h,f", [(384, 512, 1024), (333, 320, 640)], ids=["T384", "ragged_T333_h320"])
def test_one_rank_matches_the_single_gpu_stage_calls(T, h, f):
    rb, fb = binding.peer_recv_bytes(T, h, 1), binding.peer_flag_bytes(T, h, 1)
    recv, flags = _zeros_bytes(rb), _zeros_bytes(fb)
    # exchanges 1..6 on the same buffers (Y, then dX, three times), then two
    # with epoch 0, which touch no flag
    epochs = [(1, 2, 3), (3, 4, 4), (5, 6, 5), (0, 0, 6)]
    for e_y, e_dx, seed in epochs:
        inp = {k: v.cuda() for k, v in inputs.make_custom(T, h, f, seed=seed).items()}
        act = _activations(inp, inp["A"], inp["a"], inp["B"], T, h, f)
        ws = act["ws"]
        Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
        Y_ref = torch.empty_like(Y)
        q = binding.make_peer(0, 1, [recv], [flags], e_y)
        binding.mlp_tp_fc2_forward_peer(act["H"], act["H_lo"], inp["B"], T, h, f, q, ws)
        binding.mlp_tp_peer_reduce(q, inp["b"], T, h, Y, ws)
        binding.mlp_tp_fc2_forward(act["H"], act["H_lo"], inp["B"], inp["b"], T, h, f, 1, Y_ref, ws)
        binding.mlp_tp_check(ws)
        assert torch.equal(bits(Y), bits(Y_ref)), e_y
        dX = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
        dX_ref = torch.empty_like(dX)
        q = binding.make_peer(0, 1, [recv], [flags], e_dx)
        binding.mlp_tp_fc1_backward_data_peer(act["dH"], act["dH_lo"], inp["A"], T, h, f, q, ws)
        binding.mlp_tp_peer_reduce(q, None, T, h, dX, ws)
        binding.mlp_tp_fc1_backward_data(act["dH"], act["dH_lo"], inp["A"], T, h, f, 1, dX_ref, ws)
        binding.mlp_tp_check(ws)
        assert torch.equal(bits(dX), bits(dX_ref)), e_dx


@pytest.mark.parametrize("N,mode", [(2, binding.ACCURATE), (4, binding.ACCURATE), (4, binding.FAST),
                                    (8, binding.ACCURATE)], ids=["N2", "N4", "N4_fast", "N8"])
def test_emulated_ranks_sum_to_the_unsharded_block(N, mode):
    T, h, f = 512 * N // 2, 384, 2048  # T/N a multiple of 128; h ends in a ragged 256-column block
    fs = f // N
    rb, fb = binding.peer_recv_bytes(T, h, N), binding.peer_flag_bytes(T, h, N)
    assert rb == T * h * 4
    recv = [_zeros_bytes(rb) for _ in range(N)]
    flags = [_zeros_bytes(fb) for _ in range(N)]
    rows = T // N
    epoch = 0
    for seed in (7, 8):  # two forward+backward exchanges each: epochs 1..4 on the same buffers
        host = inputs.make_custom(T, h, f, seed=seed)
        inp = {k: v.cuda() for k, v in host.items()}
        ref = oracle.full(host)
        shards = [tp.shard_parameters(inp["A"], inp["a"], inp["B"], r, N) for r in range(N)]
        acts = [_activations(inp, A_i, a_i, B_i, T, h, fs) for (A_i, a_i, B_i) in shards]
        for what in ("Y", "dX"):
            epoch += 1
            qs = [binding.make_peer(r, N, recv, flags, epoch) for r in range(N)]
            for r in range(N):
                a = acts[r]
                if what == "Y":
                    lo = None if mode & binding.FAST_FC2_FORWARD else a["H_lo"]
                    binding.mlp_tp_fc2_forward_peer(a["H"], lo, shards[r][2], T, h, fs, qs[r], a["ws"])
                else:
                    lo = None if mode & binding.FAST_FC1_BACKWARD_DATA else a["dH_lo"]
                    binding.mlp_tp_fc1_backward_data_peer(a["dH"], lo, shards[r][0], T, h, fs, qs[r], a["ws"])
            outs = []
            for o in range(N):
                out = torch.empty(rows, h, dtype=torch.bfloat16, device="cuda")
                binding.mlp_tp_peer_reduce(qs[o], inp["b"] if what == "Y" else None, T, h, out, acts[o]["ws"])
                outs.append(out)
            for a in acts:
                binding.mlp_tp_check(a["ws"])
            got = torch.cat(outs, dim=0)
            assert_close(f"{what} over {N} ranks, epoch {epoch}", got, ref[what])
        # every block of every owner: 8 arrivals (epilogue warps) from each rank per exchange, consumed once
        nbl, ncb = (rows + 127) // 128, (h + 255) // 256
        for o in range(N):
            fl = flags[o].view(torch.int32).cpu().numpy()
            counters, consumed = fl[:nbl * ncb], fl[nbl * ncb:2 * nbl * ncb]
            assert np.all(counters == epoch * N * 8) and np.all(consumed == epoch), o


def _activations_fp8(inp, A_i, a_i, B_i, T, h, fs):
    """This rank's fp16 + e4m3 activations; the forward's workspace keeps the
    fp16 copy of B_i, the backward's the copy of A_i and the statistics."""
    FP8 = binding.FP8
    ws_f, ws_b = (binding.make_workspace_mode(T, h, fs, 1, FP8) for _ in range(2))
    Z = torch.empty(T, fs, dtype=torch.float32, device="cuda")
    H, dH = (torch.empty(T, fs, dtype=torch.float16, device="cuda") for _ in range(2))
    H_lo, dH_lo = (torch.empty(T, fs, dtype=torch.uint8, device="cuda") for _ in range(2))
    binding.mlp_tp_fp8_prepare_forward(B_i, T, h, fs, 1, ws_f)
    binding.mlp_tp_fc1_forward_fp8(inp["X"], A_i, a_i, T, h, fs, 1, Z, H, H_lo, ws_f)
    binding.mlp_tp_fp8_prepare_backward(inp["dY"], inp["X"], A_i, B_i, T, h, fs, 1, ws_b)
    binding.mlp_tp_fc2_backward_data_fp8(inp["dY"], B_i, Z, T, h, fs, 1, dH, dH_lo, None, ws_b)
    binding.mlp_tp_check(ws_f)
    binding.mlp_tp_check(ws_b)
    return {"H": H, "dH": dH, "ws_f": ws_f, "ws_b": ws_b}


def test_emulated_ranks_fp8_mode():
    """Four ranks in the fp16 + e4m3 mode: each rank's sH follows from its own
    shard of B, the partials leave the epilogue unscaled, and the owners' sums
    meet the bar against the unsharded block."""
    N = 4
    T, h, f = 1024, 384, 2048
    fs = f // N
    rb, fb = binding.peer_recv_bytes(T, h, N), binding.peer_flag_bytes(T, h, N)
    recv = [_zeros_bytes(rb) for _ in range(N)]
    flags = [_zeros_bytes(fb) for _ in range(N)]
    rows = T // N
    host = inputs.make_custom(T, h, f, seed=31)
    inp = {k: v.cuda() for k, v in host.items()}
    ref = oracle.full(host)
    shards = [tp.shard_parameters(inp["A"], inp["a"], inp["B"], r, N) for r in range(N)]
    acts = [_activations_fp8(inp, A_i, a_i, B_i, T, h, fs) for (A_i, a_i, B_i) in shards]
    for epoch, what in ((1, "Y"), (2, "dX")):
        qs = [binding.make_peer(r, N, recv, flags, epoch) for r in range(N)]
        for r in range(N):
            a = acts[r]
            if what == "Y":
                binding.mlp_tp_fc2_forward_peer_fp8(a["H"], T, h, fs, qs[r], a["ws_f"])
            else:
                binding.mlp_tp_fc1_backward_data_peer_fp8(a["dH"], T, h, fs, qs[r], a["ws_b"])
        outs = []
        for o in range(N):
            out = torch.empty(rows, h, dtype=torch.bfloat16, device="cuda")
            binding.mlp_tp_peer_reduce(qs[o], inp["b"] if what == "Y" else None, T, h, out, acts[o]["ws_f"])
            outs.append(out)
        for a in acts:
            binding.mlp_tp_check(a["ws_f"])
            binding.mlp_tp_check(a["ws_b"])
        assert_close(f"{what} over {N} ranks (fp8 mode)", torch.cat(outs, dim=0), ref[what])


def test_bounded_waits_report_timeout_and_the_context_survives():
    T, h, f = 256, 256, 512
    inp = {k: v.cuda() for k, v in inputs.make_custom(T, h, f, seed=9).items()}
    act = _activations(inp, inp["A"], inp["a"], inp["B"], T, h, f)
    ws = act["ws"]
    recv = _zeros_bytes(binding.peer_recv_bytes(T, h, 1))
    flags = _zeros_bytes(binding.peer_flag_bytes(T, h, 1))
    Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    try:
        binding.mlp_tp_set_wait_budget_ns(20_000_000)
        # the owner waits for arrivals of exchange 3 that nobody sends
        binding.mlp_tp_peer_reduce(binding.make_peer(0, 1, [recv], [flags], 3), inp["b"], T, h, Y, ws)
        with pytest.raises(binding.MlpError) as e:
            binding.mlp_tp_check(ws)
        assert e.value.status == 7 and "0x900" in str(e.value)
        # the writer waits for the owner to consume exchange 4, which never happened
        binding.mlp_tp_fc2_forward_peer(act["H"], act["H_lo"], inp["B"], T, h, f,
                                        binding.make_peer(0, 1, [recv], [flags], 5), ws)
        with pytest.raises(binding.MlpError) as e:
            binding.mlp_tp_check(ws)
        assert e.value.status == 7 and "0x800" in str(e.value)
    finally:
        binding.mlp_tp_set_wait_budget_ns(1_000_000_000)
    # fresh flags, epoch 1: a normal exchange on the same context
    flags.zero_()
    q = binding.make_peer(0, 1, [recv], [flags], 1)
    binding.mlp_tp_fc2_forward_peer(act["H"], act["H_lo"], inp["B"], T, h, f, q, ws)
    binding.mlp_tp_peer_reduce(q, inp["b"], T, h, Y, ws)
    binding.mlp_tp_check(ws)
    host = inputs.make_custom(T, h, f, seed=9)
    assert_close("Y after timeouts", Y, oracle.forward(host["X"], host["A"], host["a"], host["B"], host["b"])["Y"])


def _ipc_child(handle, offset, T, h, results):
    import torch as th
    from tensor_transformer_mlp_bias_b200 import binding as bd
    th.cuda.set_device(0)
    addr = bd.mlp_tp_ipc_import(handle, offset)
    out = th.empty(T, h, dtype=th.bfloat16, device="cuda")
    ws = th.zeros(256, dtype=th.uint8, device="cuda")
    bd.mlp_tp_peer_reduce(bd.make_peer(0, 1, [addr]), None, T, h, out, ws)
    bd.mlp_tp_check(ws)
    results["out"] = out.cpu().view(th.int16).numpy().tobytes()
    bd.mlp_tp_ipc_close(addr, offset)


def test_ipc_mapping_reaches_the_buffer_of_another_process():
    import torch.multiprocessing as mp
    T, h = 256, 512
    # a receive buffer inside a larger allocation: the export finds the allocation and the offset
    big = torch.zeros(4 * T * h, dtype=torch.float32, device="cuda")
    vals = torch.randn(T, h, generator=torch.Generator().manual_seed(1)).cuda()
    view = big[T * h:2 * T * h].view(T, h)
    view.copy_(vals)
    torch.cuda.synchronize()
    handle, offset = binding.mlp_tp_ipc_export(view.data_ptr())
    assert len(handle) == binding.IPC_HANDLE_BYTES and offset % 16 == 0
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    p = ctx.Process(target=_ipc_child, args=(handle, offset, T, h, results))
    p.start()
    p.join(180)
    assert p.exitcode == 0
    got = np.frombuffer(results["out"], dtype=np.int16)
    want = vals.to(torch.bfloat16).cpu().view(torch.int16).numpy().ravel()
    assert np.array_equal(got, want)


@pytest.mark.parametrize("T,world", [(300, 2), (384, 2), (64, 3)])
def test_shapes_the_token_split_cannot_serve_are_refused(T, world):
    h, fs = 256, 128
    q = binding.make_peer(0, world, [1 << 20] * world, [1 << 21] * world, 1)
    H = torch.zeros(T, fs, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(fs, h, dtype=torch.bfloat16, device="cuda")
    ws = binding.make_workspace(T, h, fs, 1)
    with pytest.raises(binding.MlpError) as e:
        binding.mlp_tp_fc2_forward_peer(H, None, B, T, h, fs, q, ws)
    assert e.value.status == 2


def test_empty_token_batch_moves_nothing():
    """T = 0: the GEMMs launch nothing and the reduce has no block; flags stay as they were."""
    h, fs = 256, 128
    for world in (1, 2):
        recv = _zeros_bytes(max(binding.peer_recv_bytes(0, h, world), 256))
        flags = _zeros_bytes(max(binding.peer_flag_bytes(0, h, world), 256))
        q = binding.make_peer(0, world, [recv] * world, [flags] * world, 1)
        B = torch.zeros(fs, h, dtype=torch.bfloat16, device="cuda")
        ws = binding.make_workspace(0, h, fs, 1)
        binding.mlp_tp_fc2_forward_peer(None, None, B, 0, h, fs, q, ws)
        binding.mlp_tp_peer_reduce(q, None, 0, h, None, ws)
        binding.mlp_tp_check(ws)
        assert int(flags.sum()) == 0
