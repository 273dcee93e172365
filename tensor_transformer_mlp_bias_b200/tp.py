"""The block sharded across GPUs: shard i of the tensor-parallel MLP on rank i.

The column/row split of "Megatron-LM — 架构与原理" (§4 巧妙之处, items
"Column→Row 配对让 MLP 只做一次通信" and "通信原语的「前向/反向对偶」")
places the column block A_i, a_i of the first layer and the row block B_i of
the second on rank i.  Each rank runs its shard through the C-ABI stage calls
with t = 1 (its shard is a whole block of width f/N).  The collectives of the
conjugate operators run between those calls:

  forward   Z_i, H_i = fc1(X, A_i, a_i)
            P_i = H_i·B_i, plus b on rank 0 only
            Y = Σ_i P_i                       all-reduce (forward of g)
  backward  dH_i = (dY·B_iᵀ) ⊙ g'(Z_i), da_i;  dB_i = H_iᵀ·dY, db
            dX = Σ_i dH_i·A_iᵀ                all-reduce (backward of f),
                                              overlapping the dA_i GEMM
            dA_i = Xᵀ·dH_i

Sequence-parallel form (the SP row of §1 它能做什么 on the same page; the SP
paragraph of "NVIDIA Megatron-LM：大规模Transformer模型分布式训练框架"): X and
dY arrive split by tokens (rank r holds rows [r·T/N, (r+1)·T/N)).  They are
all-gathered before the GEMMs, and Y and dX are reduce-scattered back to
token shards instead of all-reduced.  The GEMMs are the same.

The collectives are NCCL's (through torch.distributed) on bf16 partials, as
in the pages' system; each starts after the GEMM that produced its input.
`ops` is the object whose stage calls run the GEMMs: the C-ABI binding,
unless a caller supplies another implementation with the same signatures.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Tuple

import torch
import torch.distributed as dist

from . import binding


@dataclass
class Saved:
    """What the forward keeps for the backward on one rank."""
    X: torch.Tensor      # the full token batch (gathered in the sequence-parallel form)
    Z: torch.Tensor      # [T, f/N] pre-activation of this rank's shard
    H: torch.Tensor      # [T, f/N] activation pair of this rank's shard
    H_lo: torch.Tensor
    ws: object           # workspace of this rank's stage calls


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


def _dtypes(ops) -> Tuple[torch.dtype, torch.dtype]:
    return getattr(ops, "DTYPE", torch.bfloat16), getattr(ops, "Z_DTYPE", torch.float32)


def _gather_tokens(x: torch.Tensor, group) -> torch.Tensor:
    world = dist.get_world_size(group)
    out = torch.empty(x.shape[0] * world, *x.shape[1:], dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(out, x.contiguous(), group=group)
    return out


def _reduce_scatter_tokens(x: torch.Tensor, group, async_op: bool = False):
    world = dist.get_world_size(group)
    if x.shape[0] % world != 0:
        raise ValueError(f"T={x.shape[0]} tokens do not split over {world} ranks")
    out = torch.empty(x.shape[0] // world, *x.shape[1:], dtype=x.dtype, device=x.device)
    work = dist.reduce_scatter_tensor(out, x, group=group, async_op=async_op)
    return out, work


def forward(X: torch.Tensor, A_i: torch.Tensor, a_i: torch.Tensor, B_i: torch.Tensor, b: torch.Tensor, *,
            group=None, sequence_parallel: bool = False, mode: int = binding.ACCURATE,
            ops=binding) -> Tuple[torch.Tensor, Saved]:
    """Y (full, or this rank's token rows in the sequence-parallel form) and
    the activations the backward needs.  X is the full batch, or this rank's
    token rows in the sequence-parallel form; b is the full bias (added once,
    by rank 0)."""
    rank = dist.get_rank(group)
    if sequence_parallel:
        X = _gather_tokens(X, group)
    T, h = X.shape
    fs = A_i.shape[1]
    dt, zdt = _dtypes(ops)
    dev = X.device
    ws = ops.make_workspace(T, h, fs, 1, dev)
    Z = torch.empty(T, fs, dtype=zdt, device=dev)
    H = torch.empty(T, fs, dtype=dt, device=dev)
    H_lo = torch.empty(T, fs, dtype=dt, device=dev)
    ops.mlp_tp_fc1_forward(X, A_i, a_i, T, h, fs, 1, Z, H, H_lo, ws)
    P = torch.empty(T, h, dtype=dt, device=dev)
    ops.mlp_tp_fc2_forward(H, None if mode & binding.FAST_FC2_FORWARD else H_lo, B_i, b if rank == 0 else None,
                           T, h, fs, 1, P, ws)
    if sequence_parallel:
        Y, _ = _reduce_scatter_tokens(P, group)
    else:
        dist.all_reduce(P, group=group)
        Y = P
    return Y, Saved(X, Z, H, H_lo, ws)


def backward(dY: torch.Tensor, saved: Saved, A_i: torch.Tensor, B_i: torch.Tensor, *, group=None,
             sequence_parallel: bool = False, mode: int = binding.ACCURATE,
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
    dH, dH_lo, da = e(T, fs), e(T, fs), e(fs)
    ops.mlp_tp_fc2_backward_data(dY, B_i, saved.Z, T, h, fs, 1, dH, dH_lo, da, saved.ws)
    dB, db = e(fs, h), e(h)
    ops.mlp_tp_fc2_backward_weight(saved.H, saved.H_lo, dY, T, h, fs, 1, dB, db, saved.ws)
    Q = e(T, h)
    ops.mlp_tp_fc1_backward_data(dH, None if mode & binding.FAST_FC1_BACKWARD_DATA else dH_lo, A_i, T, h, fs, 1,
                                 Q, saved.ws)
    # the dX reduction runs while this rank computes its dA shard
    if sequence_parallel:
        dX, work = _reduce_scatter_tokens(Q, group, async_op=True)
    else:
        work = dist.all_reduce(Q, group=group, async_op=True)
        dX = Q
    dA = e(h, fs)
    ops.mlp_tp_fc1_backward_weight(saved.X, dH, dH_lo, T, h, fs, 1, dA, saved.ws)
    work.wait()
    return {"dX": dX, "dA": dA, "da": da, "dB": dB, "db": db}


def token_rows(T: int, rank: int, world: int) -> slice:
    """The token rows rank `rank` holds in the sequence-parallel form."""
    if T % world != 0:
        raise ValueError(f"T={T} tokens do not split over {world} ranks")
    n = T // world
    return slice(rank * n, (rank + 1) * n)


__all__ = ["Saved", "shard_bounds", "shard_parameters", "forward", "backward", "token_rows"]
