"""Test stand-in for the C-ABI stage calls on the CPU, in fp64, for the
multi-process tests of the cross-GPU orchestration in
tensor_transformer_mlp_bias_b200.tp.  Same call signatures as the binding.
The partial-sum calls (the *_peer GEMMs and mlp_tp_peer_reduce) support the
one-rank view the NCCL form uses: the whole partial written to slot 0 of the
caller's own buffer, which the descriptor here holds as a tensor.

It computes each stage from the oracle's definitions (GeLU and its derivative
from oracle/mlp_oracle.py, plain matrix products), writing into the output
tensors it is given.  It holds everything in fp64, so the low halves of the
activation pairs are 0.  This is test infrastructure: the library never
falls back to it.
"""
import numpy as np
import torch

from oracle import mlp_oracle as oracle

DTYPE = torch.float64
Z_DTYPE = torch.float64


def _np(x):
    return x.detach().numpy()


def make_workspace(T, h, f, t, device=None):
    return None


def mlp_tp_fc1_forward(X, A, a, T, h, f, t, Z, H, H_lo, ws, stream=None):
    z = _np(X) @ _np(A) + _np(a)
    Z.copy_(torch.from_numpy(z))
    H.copy_(torch.from_numpy(oracle.gelu(z)))
    H_lo.zero_()


def mlp_tp_fc2_forward(H, H_lo, B, b, T, h, f, t, Y, ws, stream=None):
    hh = _np(H) + (_np(H_lo) if H_lo is not None else 0.0)
    y = hh @ _np(B)
    if b is not None:
        y = y + _np(b)
    Y.copy_(torch.from_numpy(y))


def mlp_tp_fc2_backward_data(dY, B, Z, T, h, f, t, dH, dH_lo, da, ws, stream=None):
    dh = (_np(dY) @ _np(B).T) * oracle.gelu_grad(_np(Z))
    dH.copy_(torch.from_numpy(dh))
    if dH_lo is not None:
        dH_lo.zero_()
    if da is not None:
        da.copy_(torch.from_numpy(dh.sum(axis=0)))


def mlp_tp_fc2_backward_weight(H, H_lo, dY, T, h, f, t, dB, db, ws, stream=None):
    hh = _np(H) + (_np(H_lo) if H_lo is not None else 0.0)
    dB.copy_(torch.from_numpy(hh.T @ _np(dY)))
    if db is not None:
        db.copy_(torch.from_numpy(_np(dY).sum(axis=0)))


def mlp_tp_fc1_backward_data(dH, dH_lo, A, T, h, f, t, dX, ws, stream=None):
    dh = _np(dH) + (_np(dH_lo) if dH_lo is not None else 0.0)
    dX.copy_(torch.from_numpy(dh @ _np(A).T))


def mlp_tp_fc1_backward_weight(X, dH, dH_lo, T, h, f, t, dA, ws, stream=None):
    dh = _np(dH) + (_np(dH_lo) if dH_lo is not None else 0.0)
    dA.copy_(torch.from_numpy(np.asarray(_np(X)).T @ dh))


class _Peer:
    def __init__(self, rank, world, recv, flags=None, epoch=0):
        if world != 1 or epoch != 0:
            raise NotImplementedError("the CPU stand-in has no cross-process buffers")
        self.rank, self.world, self.recv, self.epoch = rank, world, list(recv), epoch


def make_peer(rank, world, recv, flags=None, epoch=0):
    return _Peer(rank, world, recv, flags, epoch)


def mlp_tp_fc2_forward_peer(H, H_lo, B, T, h, fs, peer, ws, stream=None):
    hh = _np(H) + (_np(H_lo) if H_lo is not None else 0.0)
    peer.recv[0].copy_(torch.from_numpy(hh @ _np(B)))


def mlp_tp_fc1_backward_data_peer(dH, dH_lo, A, T, h, fs, peer, ws, stream=None):
    dh = _np(dH) + (_np(dH_lo) if dH_lo is not None else 0.0)
    peer.recv[0].copy_(torch.from_numpy(dh @ _np(A).T))


def mlp_tp_peer_reduce(peer, bias, T, h, out, ws, stream=None):
    s = _np(peer.recv[0])[:T]
    out.copy_(torch.from_numpy(s + (_np(bias) if bias is not None else 0.0)))


# ---- the fp16 + e4m3 mode's calls (the library keeps dH scaled by a power of
# two between its stages; this stand-in keeps the scale 1, all in fp64)
F16_DTYPE = torch.float64
E4M3_DTYPE = torch.float64


def make_workspace_mode(T, h, f, t, mode, recompute=False, device=None):
    return {}  # the prepare calls leave the weight and input copies here


def mlp_tp_fp8_prepare_forward(B, T, h, f, t, ws, stream=None):
    ws["B"] = B


def mlp_tp_fp8_prepare_backward(dY, X, A, B, T, h, f, t, ws, stream=None):
    ws["A"], ws["X"] = A, X


def mlp_tp_fc1_forward_fp8(X, A, a, T, h, f, t, Z, H, H_lo, ws, stream=None):
    mlp_tp_fc1_forward(X, A, a, T, h, f, t, Z, H, H_lo, ws)


def mlp_tp_fc2_forward_peer_fp8(H, T, h, fs, peer, ws, stream=None):
    peer.recv[0].copy_(torch.from_numpy(_np(H) @ _np(ws["B"])))


def mlp_tp_fc2_backward_data_fp8(dY, B, Z, T, h, f, t, dH, dH_lo, da, ws, stream=None):
    mlp_tp_fc2_backward_data(dY, B, Z, T, h, f, t, dH, dH_lo, da, ws)


def mlp_tp_fc2_backward_weight_fp8(H, H_lo, dY, T, h, f, t, dB, db, ws, stream=None):
    mlp_tp_fc2_backward_weight(H, H_lo, dY, T, h, f, t, dB, db, ws)


def mlp_tp_fc1_backward_data_peer_fp8(dH, T, h, fs, peer, ws, stream=None):
    peer.recv[0].copy_(torch.from_numpy(_np(dH) @ _np(ws["A"]).T))


def mlp_tp_fc1_backward_weight_fp8(dH, dH_lo, T, h, f, t, dA, ws, stream=None):
    mlp_tp_fc1_backward_weight(ws["X"], dH, dH_lo, T, h, f, t, dA, ws)
