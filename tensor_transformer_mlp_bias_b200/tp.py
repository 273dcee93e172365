"""The block sharded across GPUs: shard i of the tensor-parallel MLP on rank i.

The column/row split of "Megatron-LM — 架构与原理" (§4 巧妙之处, items
"Column→Row 配对让 MLP 只做一次通信" and "通信原语的「前向/反向对偶」")
places the column block A_i, a_i of the first layer and the row block B_i of
the second on rank i.  Each rank runs its shard through the C-ABI stage calls
with t = 1 (its shard is a whole block of width f/N).  The sums of the
conjugate operators run between those calls:

  forward   Z_i, H_i = fc1(X, A_i, a_i)
            P_i = H_i·B_i                     (fp32)
            Y = Σ_i P_i + b                   reduce's forward all-reduce
  backward  dH_i = (dY·B_iᵀ) ⊙ g'(Z_i), da_i;  dB_i = H_iᵀ·dY, db
            Q_i = dH_i·A_iᵀ                   (fp32)
            dX = Σ_i Q_i                      copy's backward all-reduce
            dA_i = Xᵀ·dH_i

The partials stay fp32 and the sum is rounded once: a 16-bit all-reduce of
each rank's rounded output misses the parity bar on the 8.3B-class workload
(tests/test_tp_precision.py).  Two ways to form the sum:

  reduction="peer" (default)  the fused form.  The row-parallel GEMM's
      epilogue stores each 128-row block of its fp32 partial straight into
      the buffer of the rank that owns those tokens (CUDA IPC mappings over
      NVLink), and that rank's reduce kernel adds the N partials in rank
      order plus b and rounds once: a reduce-scatter inside the GEMM.  The
      plain tensor-parallel form then all-gathers the bf16 rows (NCCL).
  reduction="nccl"  the baseline: the GEMM writes its fp32 partial locally,
      NCCL all-reduces (or reduce-scatters) it in fp32, and the same reduce
      kernel adds b and rounds once.

Sequence-parallel form (the SP row of §1 它能做什么 on the same page; the SP
paragraph of "NVIDIA Megatron-LM：大规模Transformer模型分布式训练框架"): X and
dY arrive split by tokens (rank r holds rows [r·T/N, (r+1)·T/N)).  They are
all-gathered before the GEMMs, and Y and dX stay split by tokens: the
reduce-scatter alone.

Precision modes: as the composite calls (mode=binding.ACCURATE by default).
With binding.FP8 each rank runs the fp16 + e4m3 stage calls on its shard: the
prepare calls cast its B_i (forward) and X, dY, A_i (backward) in its own
workspace, and the row-parallel GEMMs send unscaled fp32 partials (each rank
undoes its own dH scale), so the reduction is the same in every mode.

`ops` is the object whose stage calls run the GEMMs: the C-ABI binding,
unless a caller supplies another implementation with the same signatures.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import torch
import torch.distributed as dist

from . import binding


def exchange_addresses(own_ptr: int, group=None, ops=binding) -> Tuple[List[int], List[Tuple[int, int]]]:
    """Every rank's buffer as addressed from this process: this rank's own
    pointer for itself, a CUDA IPC mapping of each other rank's.  Returns the
    table and the (address, offset) pairs this process mapped (to unmap)."""
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    if world == 1:
        return [own_ptr], []
    mine = ops.mlp_tp_ipc_export(own_ptr)
    every = [None] * world
    dist.all_gather_object(every, mine, group=group)
    table, mapped = [], []
    for r in range(world):
        if r == rank:
            table.append(own_ptr)
        else:
            handle, offset = every[r]
            addr = ops.mlp_tp_ipc_import(handle, offset)
            table.append(addr)
            mapped.append((addr, offset))
    return table, mapped


class PeerExchange:
    """One rank's receive buffer and flag block of the fused cross-GPU
    reduction, the table of every rank's buffers as addressed from this GPU,
    and the exchange counter (epoch) the ranks advance together.  One object
    serves any number of exchanges of [T, h] partials in sequence (the Y of a
    forward, then the dX of its backward, ...).  Created collectively by every
    rank of the group."""

    def __init__(self, T: int, h: int, group=None, device=None, ops=binding):
        self.world, self.rank = dist.get_world_size(group), dist.get_rank(group)
        self.T, self.h, self.ops = T, h, ops
        self.recv_bytes = ops.peer_recv_bytes(T, h, self.world)
        self.flag_bytes = ops.peer_flag_bytes(T, h, self.world)
        if self.recv_bytes == 0 or self.flag_bytes == 0:
            raise ValueError(f"no cross-GPU buffers for T={T} h={h} over {self.world} ranks")
        # receive buffer and flag block in one allocation: one IPC mapping per peer
        self.buf = torch.zeros(self.recv_bytes + self.flag_bytes, dtype=torch.uint8, device=device)
        self.table, self._mapped = exchange_addresses(self.buf.data_ptr(), group, ops)
        self.epoch = 0

    def next(self):
        """The descriptor of the next exchange (epoch + 1)."""
        self.epoch += 1
        return self.ops.make_peer(self.rank, self.world, self.table,
                                  [a + self.recv_bytes for a in self.table], self.epoch)

    def close(self):
        for addr, offset in self._mapped:
            self.ops.mlp_tp_ipc_close(addr, offset)
        self._mapped = []


@dataclass
class Saved:
    """What the forward keeps for the backward on one rank."""
    X: torch.Tensor      # the full token batch (gathered in the sequence-parallel form)
    Z: torch.Tensor      # [T, f/N] pre-activation of this rank's shard
    H: torch.Tensor      # [T, f/N] activation pair of this rank's shard
    H_lo: torch.Tensor
    ws: object           # workspace of this rank's stage calls
    exchange: Optional[PeerExchange] = None
    owns_exchange: bool = False  # created by forward(): the backward closes it


def shard_bounds(f: int, rank: int, world: int) -> Tuple[int, int]:
    """Columns of A and a, rows of B, held by `rank`."""
    if f % world != 0:
        raise ValueError(f"f={f} is not divisible by the {world} ranks")
    fs = f // world
    return rank * fs, (rank + 1) * fs


def shard_parameters(A: torch.Tensor, a: torch.Tensor, B: torch.Tensor, rank: int,
                     world: int) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Rank `rank`'s column block of A and a and row block of B (contiguous copies)."""
    lo, hi = shard_bounds(A.shape[1], rank, world)
    return A[:, lo:hi].contiguous(), a[lo:hi].contiguous(), B[lo:hi, :].contiguous()


def token_rows(T: int, rank: int, world: int) -> slice:
    """The token rows rank `rank` holds in the sequence-parallel form (and owns in the reduce-scatter)."""
    if T % world != 0:
        raise ValueError(f"T={T} tokens do not split over {world} ranks")
    n = T // world
    return slice(rank * n, (rank + 1) * n)


def _dtypes(ops) -> Tuple[torch.dtype, torch.dtype]:
    return getattr(ops, "DTYPE", torch.bfloat16), getattr(ops, "Z_DTYPE", torch.float32)


def _fp8_dtypes(ops) -> Tuple[torch.dtype, torch.dtype]:
    """Element types of the fp16 + e4m3 mode's activations (fp16 value, e4m3 residual)."""
    return getattr(ops, "F16_DTYPE", torch.float16), getattr(ops, "E4M3_DTYPE", torch.uint8)


def _gather_tokens(x: torch.Tensor, group) -> torch.Tensor:
    world = dist.get_world_size(group)
    out = torch.empty(x.shape[0] * world, *x.shape[1:], dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(out, x.contiguous(), group=group)
    return out


def _sum_partials(gemm, bias, T: int, h: int, dev, *, group, sequence_parallel: bool, reduction: str,
                  exchange: Optional[PeerExchange], ws, ops):
    """Σ over ranks of this rank's fp32 partial (produced by `gemm(peer)`),
    plus `bias`, rounded once: this rank's token rows in the sequence-parallel
    form, all T rows otherwise."""
    world = dist.get_world_size(group)
    dt, _ = _dtypes(ops)
    rows = T // world
    if reduction == "peer":
        q = exchange.next()
        gemm(q)
        out_rows = torch.empty(rows, h, dtype=dt, device=dev)
        ops.mlp_tp_peer_reduce(q, bias, T, h, out_rows, ws)
        return out_rows if sequence_parallel else _gather_tokens(out_rows, group)
    if reduction != "nccl":
        raise ValueError(f"unknown reduction {reduction!r}")
    P = torch.empty(T, h, dtype=torch.float32 if dt == torch.bfloat16 else dt, device=dev)
    gemm(ops.make_peer(0, 1, [P]))           # the whole fp32 partial, locally
    if sequence_parallel:
        S = torch.empty(rows, h, dtype=P.dtype, device=dev)
        dist.reduce_scatter_tensor(S, P, group=group)
        out = torch.empty(rows, h, dtype=dt, device=dev)
        ops.mlp_tp_peer_reduce(ops.make_peer(0, 1, [S]), bias, rows, h, out, ws)
        return out
    dist.all_reduce(P, group=group)
    out = torch.empty(T, h, dtype=dt, device=dev)
    ops.mlp_tp_peer_reduce(ops.make_peer(0, 1, [P]), bias, T, h, out, ws)
    return out


def forward(X: torch.Tensor, A_i: torch.Tensor, a_i: torch.Tensor, B_i: torch.Tensor, b: torch.Tensor, *,
            group=None, sequence_parallel: bool = False, mode: int = binding.ACCURATE, reduction: str = "peer",
            exchange: Optional[PeerExchange] = None, ops=binding) -> Tuple[torch.Tensor, Saved]:
    """Y (full, or this rank's token rows in the sequence-parallel form) and
    the activations the backward needs.  X is the full batch, or this rank's
    token rows in the sequence-parallel form; b is the full bias (added once,
    to the summed partials).  With reduction="peer", `exchange` is the
    group's PeerExchange for [T, h] partials (created here when None)."""
    if sequence_parallel:
        X = _gather_tokens(X, group)
    T, h = X.shape
    fs = A_i.shape[1]
    dt, zdt = _dtypes(ops)
    dev = X.device
    owns = reduction == "peer" and exchange is None
    if owns:
        exchange = PeerExchange(T, h, group, dev, ops)
    Z = torch.empty(T, fs, dtype=zdt, device=dev)
    if mode == binding.FP8:
        # fp16 H with its e4m3 residual; the fp16 copy of B_i lives in the workspace
        ws = ops.make_workspace_mode(T, h, fs, 1, binding.FP8, device=dev)
        f16, e4m3 = _fp8_dtypes(ops)
        H = torch.empty(T, fs, dtype=f16, device=dev)
        H_lo = torch.empty(T, fs, dtype=e4m3, device=dev)
        ops.mlp_tp_fp8_prepare_forward(B_i, T, h, fs, 1, ws)
        ops.mlp_tp_fc1_forward_fp8(X, A_i, a_i, T, h, fs, 1, Z, H, H_lo, ws)
        gemm = lambda q: ops.mlp_tp_fc2_forward_peer_fp8(H, T, h, fs, q, ws)  # noqa: E731
    else:
        ws = ops.make_workspace(T, h, fs, 1, dev)
        H = torch.empty(T, fs, dtype=dt, device=dev)
        H_lo = torch.empty(T, fs, dtype=dt, device=dev)
        ops.mlp_tp_fc1_forward(X, A_i, a_i, T, h, fs, 1, Z, H, H_lo, ws)
        lo = None if mode & binding.FAST_FC2_FORWARD else H_lo
        gemm = lambda q: ops.mlp_tp_fc2_forward_peer(H, lo, B_i, T, h, fs, q, ws)  # noqa: E731
    Y = _sum_partials(gemm, b, T, h, dev, group=group, sequence_parallel=sequence_parallel, reduction=reduction,
                      exchange=exchange, ws=ws, ops=ops)
    return Y, Saved(X, Z, H, H_lo, ws, exchange, owns)


def backward(dY: torch.Tensor, saved: Saved, A_i: torch.Tensor, B_i: torch.Tensor, *, group=None,
             sequence_parallel: bool = False, mode: int = binding.ACCURATE, reduction: str = "peer",
             ops=binding) -> Dict[str, torch.Tensor]:
    """dX (full, or this rank's token rows in the sequence-parallel form), this
    rank's shard of dA, da and dB, and db.  dY is the full gradient, or this
    rank's token rows in the sequence-parallel form."""
    if sequence_parallel:
        dY = _gather_tokens(dY, group)
    T, h = dY.shape
    fs = A_i.shape[1]
    dt, _ = _dtypes(ops)
    dev = dY.device
    e = lambda *s: torch.empty(*s, dtype=dt, device=dev)  # noqa: E731
    da, dB, db = e(fs), e(fs, h), e(h)
    fp8 = mode == binding.FP8
    if fp8:
        # statistics, scales and the fp16 / e4m3 copies of X, dY and A_i in the workspace
        f16, e4m3 = _fp8_dtypes(ops)
        dH = torch.empty(T, fs, dtype=f16, device=dev)
        dH_lo = torch.empty(T, fs, dtype=e4m3, device=dev)
        ops.mlp_tp_fp8_prepare_backward(dY, saved.X, A_i, B_i, T, h, fs, 1, saved.ws)
        ops.mlp_tp_fc2_backward_data_fp8(dY, B_i, saved.Z, T, h, fs, 1, dH, dH_lo, da, saved.ws)
        ops.mlp_tp_fc2_backward_weight_fp8(saved.H, saved.H_lo, dY, T, h, fs, 1, dB, db, saved.ws)
        gemm = lambda q: ops.mlp_tp_fc1_backward_data_peer_fp8(dH, T, h, fs, q, saved.ws)  # noqa: E731
    else:
        dH, dH_lo = e(T, fs), e(T, fs)
        ops.mlp_tp_fc2_backward_data(dY, B_i, saved.Z, T, h, fs, 1, dH, dH_lo, da, saved.ws)
        ops.mlp_tp_fc2_backward_weight(saved.H, saved.H_lo, dY, T, h, fs, 1, dB, db, saved.ws)
        lo = None if mode & binding.FAST_FC1_BACKWARD_DATA else dH_lo
        gemm = lambda q: ops.mlp_tp_fc1_backward_data_peer(dH, lo, A_i, T, h, fs, q, saved.ws)  # noqa: E731
    exchange, owns = saved.exchange, saved.owns_exchange
    if reduction == "peer" and exchange is None:
        exchange, owns = PeerExchange(T, h, group, dev, ops), True
    dX = _sum_partials(gemm, None, T, h, dev, group=group, sequence_parallel=sequence_parallel,
                       reduction=reduction, exchange=exchange, ws=saved.ws, ops=ops)
    dA = e(h, fs)
    if fp8:
        ops.mlp_tp_fc1_backward_weight_fp8(dH, dH_lo, T, h, fs, 1, dA, saved.ws)
    else:
        ops.mlp_tp_fc1_backward_weight(saved.X, dH, dH_lo, T, h, fs, 1, dA, saved.ws)
    if owns:
        # the exchange's buffers are read by this rank's last reduce and by the
        # other ranks' GEMMs: every rank syncs and meets before it unmaps
        if dev.type == "cuda":
            torch.cuda.synchronize(dev)
        dist.barrier(group=group)
        exchange.close()
    return {"dX": dX, "dA": dA, "da": da, "dB": dB, "db": db}


__all__ = ["PeerExchange", "Saved", "exchange_addresses", "shard_bounds", "shard_parameters", "forward", "backward",
           "token_rows"]
