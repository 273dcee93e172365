"""ctypes binding of the C-ABI library ``libmlptp.so`` (include/mlp_tp.h).

Argument marshalling only: every function here takes torch tensors (or raw
integer device addresses), checks that tensors are contiguous bf16 CUDA
tensors, passes their addresses and the stream to the C entry point of the
same name, and raises :class:`MlpError` on a non-OK status.  All arithmetic
runs in the library's kernels.  The library is loaded on first use; if it
has not been built, the call raises (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmlptp.so")

STATUS = {
    0: "MLP_OK",
    1: "MLP_ERR_INVALID_ARG",
    2: "MLP_ERR_UNSUPPORTED_SHAPE",
    3: "MLP_ERR_MISALIGNED",
    4: "MLP_ERR_WORKSPACE_TOO_SMALL",
    5: "MLP_ERR_UNSUPPORTED_DEVICE",
    6: "MLP_ERR_CUDA",
    7: "MLP_ERR_TIMEOUT",
    8: "MLP_ERR_BOUNDS",
    9: "MLP_ERR_RANGE",
}

# name -> argument ctypes, in header order
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t

MAX_WORLD = 8
IPC_HANDLE_BYTES = 64


class Peer(ctypes.Structure):
    """mlp_tp_peer_t: one rank's view of the cross-GPU reduction buffers."""
    _fields_ = [("rank", ctypes.c_int32), ("world", ctypes.c_int32), ("epoch", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32), ("recv", ctypes.c_void_p * MAX_WORLD),
                ("flags", ctypes.c_void_p * MAX_WORLD)]


_PP = ctypes.POINTER(Peer)
_SIGS = {
    "mlp_tp_workspace_bytes": ([_I64, _I64, _I64, _I32], _SZ),
    "mlp_tp_forward": ([_P] * 5 + [_I64, _I64, _I64, _I32, _I32] + [_P] * 4 + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc1_forward": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] * 3 + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc2_forward": ([_P] * 4 + [_I64, _I64, _I64, _I32] + [_P] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_backward": ([_P] * 7 + [_I64, _I64, _I64, _I32, _I32] + [_P] * 5 + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc2_backward_data": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] * 3 + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc2_backward_weight": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] * 2 + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc1_backward_data": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc1_backward_weight": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_recompute_workspace_bytes": ([_I64, _I64, _I64, _I32], _SZ),
    "mlp_tp_forward_recompute": ([_P] * 5 + [_I64, _I64, _I64, _I32, _I32] + [_P] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_backward_recompute": ([_P] * 5 + [_I64, _I64, _I64, _I32, _I32] + [_P] * 5 + [_P, _SZ, _P],
                                  ctypes.c_int),
    "mlp_tp_workspace_bytes_mode": ([_I64, _I64, _I64, _I32, _I32], _SZ),
    "mlp_tp_recompute_workspace_bytes_mode": ([_I64, _I64, _I64, _I32, _I32], _SZ),
    "mlp_tp_fp8_prepare_forward": ([_P] + [_I64, _I64, _I64, _I32] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fp8_prepare_backward": ([_P] * 4 + [_I64, _I64, _I64, _I32] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc1_forward_fp8": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] * 3 + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc2_forward_fp8": ([_P] * 2 + [_I64, _I64, _I64, _I32] + [_P] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc2_backward_data_fp8": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] * 3 + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc2_backward_weight_fp8": ([_P] * 3 + [_I64, _I64, _I64, _I32] + [_P] * 2 + [_P, _SZ, _P],
                                       ctypes.c_int),
    "mlp_tp_fc1_backward_data_fp8": ([_P] + [_I64, _I64, _I64, _I32] + [_P] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc1_backward_weight_fp8": ([_P] * 2 + [_I64, _I64, _I64, _I32] + [_P] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_peer_recv_bytes": ([_I64, _I64, _I32], _SZ),
    "mlp_tp_peer_flag_bytes": ([_I64, _I64, _I32], _SZ),
    "mlp_tp_fc2_forward_peer": ([_P] * 3 + [_I64] * 3 + [_PP] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc1_backward_data_peer": ([_P] * 3 + [_I64] * 3 + [_PP] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc2_forward_peer_fp8": ([_P] + [_I64] * 3 + [_PP] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_fc1_backward_data_peer_fp8": ([_P] + [_I64] * 3 + [_PP] + [_P, _SZ, _P], ctypes.c_int),
    "mlp_tp_peer_reduce": ([_PP, _P, _I64, _I64, _P, _P, _SZ, _P], ctypes.c_int),
    "mlp_tp_ipc_export": ([_P, _P, ctypes.POINTER(ctypes.c_uint64)], ctypes.c_int),
    "mlp_tp_ipc_import": ([_P, ctypes.c_uint64, ctypes.POINTER(_P)], ctypes.c_int),
    "mlp_tp_ipc_close": ([_P, ctypes.c_uint64], ctypes.c_int),
    "mlp_tp_fc2_bias_grad_noalloc": ([_P, _I64, _I64, _P, _P], ctypes.c_int),
    "mlp_tp_check": ([_P, _P], ctypes.c_int),
    "mlp_tp_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "mlp_tp_last_error": ([], ctypes.c_char_p),
    "mlp_tp_launch_count": ([], ctypes.c_uint64),
    "mlp_tp_set_wait_budget_ns": ([ctypes.c_uint64], None),
    "mlp_tp_set_debug_flags": ([ctypes.c_uint32], None),
}

# precision modes of the composite calls (mlp_tp_mode_t); 0 is the accurate default
ACCURATE = 0
FAST_FC2_FORWARD = 1
FAST_FC1_BACKWARD_DATA = 2
FAST = 3
FP8 = 4  # fp16 operands with e4m3 residual products; H, dH fp16 and H_lo, dH_lo e4m3

_lib: Optional[ctypes.CDLL] = None


class MlpError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libmlptp.so (once).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; run `python -m tensor_transformer_mlp_bias_b200.build` "
                "(the CUDA library is the only implementation; there is no fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def exported_symbols():
    return list(_SIGS)


# ------------------------------------------------------------------ marshalling
def _addr(x, name: str, nullable: bool = False, fmt: str = None):
    """Device address of `x`.  `fmt` overrides the expected element type:
    "f16" (fp16) or "e4m3" (one byte per value: uint8 or float8_e4m3fn)."""
    if x is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if isinstance(x, int):
        return x
    import torch
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor or an int address")
    if x.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {x.device})")
    if fmt == "e4m3":
        want = (torch.uint8, torch.float8_e4m3fn)
    elif fmt == "f16":
        want = (torch.float16,)
    else:
        want = (torch.float32,) if name == "Z" else (torch.bfloat16,)
    if name != "ws" and x.dtype not in want:
        raise ValueError(f"{name} must be {' or '.join(str(w) for w in want)} (got {x.dtype})")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ws(ws):
    import torch
    if isinstance(ws, torch.Tensor):
        return _addr(ws, "ws"), ws.numel() * ws.element_size()
    addr, nbytes = ws
    return addr, nbytes


def _check(status: int):
    if status != 0:
        msg = lib().mlp_tp_last_error()
        raise MlpError(status, msg.decode() if msg else "")


def workspace_bytes(T: int, h: int, f: int, t: int) -> int:
    return int(lib().mlp_tp_workspace_bytes(T, h, f, t))


def make_workspace(T: int, h: int, f: int, t: int, device="cuda"):
    """Zero-filled uint8 device workspace (torch allocations are 256-byte aligned)."""
    import torch
    n = workspace_bytes(T, h, f, t)
    if n == 0:
        raise MlpError(2, f"unsupported shape T={T} h={h} f={f} t={t}")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _h_fmts(mode):
    """Element types of (H, H_lo) and (dH, dH_lo) in a precision mode."""
    return ("f16", "e4m3") if mode == FP8 else (None, None)


def mlp_tp_forward(X, A, a, B, b, T, h, f, t, mode, Y, Z, H, H_lo, ws, stream=None):
    w, wn = _ws(ws)
    fh, fl = _h_fmts(mode)
    _check(lib().mlp_tp_forward(_addr(X, "X"), _addr(A, "A"), _addr(a, "a"), _addr(B, "B"), _addr(b, "b"),
                                T, h, f, t, mode, _addr(Y, "Y"), _addr(Z, "Z"), _addr(H, "H", fmt=fh),
                                _addr(H_lo, "H_lo", fmt=fl), w, wn, _stream(stream)))


def mlp_tp_fc1_forward(X, A, a, T, h, f, t, Z, H, H_lo, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_forward(_addr(X, "X"), _addr(A, "A"), _addr(a, "a"), T, h, f, t,
                                    _addr(Z, "Z"), _addr(H, "H"), _addr(H_lo, "H_lo"), w, wn, _stream(stream)))


def mlp_tp_fc2_forward(H, H_lo, B, b, T, h, f, t, Y, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_forward(_addr(H, "H"), _addr(H_lo, "H_lo", True), _addr(B, "B"), _addr(b, "b", True),
                                    T, h, f, t, _addr(Y, "Y"), w, wn, _stream(stream)))


def mlp_tp_backward(dY, X, A, B, Z, H, H_lo, T, h, f, t, mode, dX, dA, da, dB, db, ws, stream=None):
    w, wn = _ws(ws)
    fh, fl = _h_fmts(mode)
    _check(lib().mlp_tp_backward(_addr(dY, "dY"), _addr(X, "X"), _addr(A, "A"), _addr(B, "B"), _addr(Z, "Z"),
                                 _addr(H, "H", fmt=fh), _addr(H_lo, "H_lo", fmt=fl), T, h, f, t, mode,
                                 _addr(dX, "dX"),
                                 _addr(dA, "dA"), _addr(da, "da", True), _addr(dB, "dB"), _addr(db, "db", True),
                                 w, wn, _stream(stream)))


def mlp_tp_fc2_backward_data(dY, B, Z, T, h, f, t, dH, dH_lo, da, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_backward_data(_addr(dY, "dY"), _addr(B, "B"), _addr(Z, "Z"), T, h, f, t,
                                          _addr(dH, "dH"), _addr(dH_lo, "dH_lo"), _addr(da, "da", True),
                                          w, wn, _stream(stream)))


def mlp_tp_fc2_backward_weight(H, H_lo, dY, T, h, f, t, dB, db, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_backward_weight(_addr(H, "H"), _addr(H_lo, "H_lo"), _addr(dY, "dY"), T, h, f, t,
                                            _addr(dB, "dB"), _addr(db, "db", True), w, wn, _stream(stream)))


def mlp_tp_fc1_backward_data(dH, dH_lo, A, T, h, f, t, dX, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_backward_data(_addr(dH, "dH"), _addr(dH_lo, "dH_lo", True), _addr(A, "A"),
                                          T, h, f, t, _addr(dX, "dX"), w, wn, _stream(stream)))


def mlp_tp_fc1_backward_weight(X, dH, dH_lo, T, h, f, t, dA, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_backward_weight(_addr(X, "X"), _addr(dH, "dH"), _addr(dH_lo, "dH_lo"), T, h, f, t,
                                            _addr(dA, "dA"), w, wn, _stream(stream)))


def recompute_workspace_bytes(T: int, h: int, f: int, t: int) -> int:
    return int(lib().mlp_tp_recompute_workspace_bytes(T, h, f, t))


def make_recompute_workspace(T: int, h: int, f: int, t: int, device="cuda"):
    import torch
    n = recompute_workspace_bytes(T, h, f, t)
    if n == 0:
        raise MlpError(2, f"unsupported shape T={T} h={h} f={f} t={t}")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def mlp_tp_forward_recompute(X, A, a, B, b, T, h, f, t, mode, Y, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_forward_recompute(_addr(X, "X", T == 0), _addr(A, "A"), _addr(a, "a"), _addr(B, "B"),
                                          _addr(b, "b"), T, h, f, t, mode, _addr(Y, "Y", T == 0), w, wn,
                                          _stream(stream)))


def mlp_tp_backward_recompute(dY, X, A, a, B, T, h, f, t, mode, dX, dA, da, dB, db, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_backward_recompute(_addr(dY, "dY", T == 0), _addr(X, "X", T == 0), _addr(A, "A"),
                                           _addr(a, "a"), _addr(B, "B"), T, h, f, t, mode,
                                           _addr(dX, "dX", T == 0), _addr(dA, "dA"), _addr(da, "da", True),
                                           _addr(dB, "dB"), _addr(db, "db", True), w, wn, _stream(stream)))


def workspace_bytes_mode(T: int, h: int, f: int, t: int, mode: int) -> int:
    return int(lib().mlp_tp_workspace_bytes_mode(T, h, f, t, mode))


def recompute_workspace_bytes_mode(T: int, h: int, f: int, t: int, mode: int) -> int:
    return int(lib().mlp_tp_recompute_workspace_bytes_mode(T, h, f, t, mode))


def make_workspace_mode(T: int, h: int, f: int, t: int, mode: int, recompute: bool = False, device="cuda"):
    """Zero-filled workspace for a precision mode (MLP_TP_FP8 needs more)."""
    import torch
    n = (recompute_workspace_bytes_mode if recompute else workspace_bytes_mode)(T, h, f, t, mode)
    if n == 0:
        raise MlpError(2, f"unsupported shape or mode T={T} h={h} f={f} t={t} mode={mode}")
    return torch.zeros(n, dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ the fp16 + e4m3 mode by stage
def mlp_tp_fp8_prepare_forward(B, T, h, f, t, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fp8_prepare_forward(_addr(B, "B"), T, h, f, t, w, wn, _stream(stream)))


def mlp_tp_fp8_prepare_backward(dY, X, A, B, T, h, f, t, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fp8_prepare_backward(_addr(dY, "dY", T == 0), _addr(X, "X", T == 0), _addr(A, "A"),
                                             _addr(B, "B"), T, h, f, t, w, wn, _stream(stream)))


def mlp_tp_fc1_forward_fp8(X, A, a, T, h, f, t, Z, H, H_lo, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_forward_fp8(_addr(X, "X", T == 0), _addr(A, "A"), _addr(a, "a"), T, h, f, t,
                                        _addr(Z, "Z", T == 0), _addr(H, "H", T == 0, "f16"),
                                        _addr(H_lo, "H_lo", T == 0, "e4m3"), w, wn, _stream(stream)))


def mlp_tp_fc2_forward_fp8(H, b, T, h, f, t, Y, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_forward_fp8(_addr(H, "H", T == 0, "f16"), _addr(b, "b", True), T, h, f, t,
                                        _addr(Y, "Y", T == 0), w, wn, _stream(stream)))


def mlp_tp_fc2_backward_data_fp8(dY, B, Z, T, h, f, t, dH, dH_lo, da, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_backward_data_fp8(_addr(dY, "dY", T == 0), _addr(B, "B"), _addr(Z, "Z", T == 0),
                                              T, h, f, t, _addr(dH, "dH", T == 0, "f16"),
                                              _addr(dH_lo, "dH_lo", T == 0, "e4m3"), _addr(da, "da", True),
                                              w, wn, _stream(stream)))


def mlp_tp_fc2_backward_weight_fp8(H, H_lo, dY, T, h, f, t, dB, db, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_backward_weight_fp8(_addr(H, "H", T == 0, "f16"), _addr(H_lo, "H_lo", T == 0, "e4m3"),
                                                _addr(dY, "dY", T == 0), T, h, f, t, _addr(dB, "dB"),
                                                _addr(db, "db", True), w, wn, _stream(stream)))


def mlp_tp_fc1_backward_data_fp8(dH, T, h, f, t, dX, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_backward_data_fp8(_addr(dH, "dH", T == 0, "f16"), T, h, f, t, _addr(dX, "dX", T == 0),
                                              w, wn, _stream(stream)))


def mlp_tp_fc1_backward_weight_fp8(dH, dH_lo, T, h, f, t, dA, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_backward_weight_fp8(_addr(dH, "dH", T == 0, "f16"),
                                                _addr(dH_lo, "dH_lo", T == 0, "e4m3"), T, h, f, t,
                                                _addr(dA, "dA"), w, wn, _stream(stream)))


# ------------------------------------------------------------------ across GPUs
def _ptr(x):
    if x is None:
        return None
    return x if isinstance(x, int) else x.data_ptr()


def make_peer(rank: int, world: int, recv, flags=None, epoch: int = 0) -> Peer:
    """mlp_tp_peer_t for rank `rank` of `world`: recv[o] and flags[o] are rank
    o's receive buffer and flag block as addressed from this GPU (ints or
    tensors; flags may be None when epoch == 0)."""
    if not 1 <= world <= MAX_WORLD or not 0 <= rank < world or len(recv) != world:
        raise ValueError(f"peer table: rank {rank} of {world} with {len(recv)} buffers")
    p = Peer()
    p.rank, p.world, p.epoch, p.reserved = rank, world, epoch, 0
    for o in range(world):
        p.recv[o] = _ptr(recv[o])
        p.flags[o] = _ptr(flags[o]) if flags is not None else None
    return p


def peer_recv_bytes(T: int, h: int, world: int) -> int:
    return int(lib().mlp_tp_peer_recv_bytes(T, h, world))


def peer_flag_bytes(T: int, h: int, world: int) -> int:
    return int(lib().mlp_tp_peer_flag_bytes(T, h, world))


def mlp_tp_fc2_forward_peer(H, H_lo, B, T, h, fs, peer: Peer, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_forward_peer(_addr(H, "H", T == 0), _addr(H_lo, "H_lo", True), _addr(B, "B"), T, h, fs,
                                         ctypes.byref(peer), w, wn, _stream(stream)))


def mlp_tp_fc1_backward_data_peer(dH, dH_lo, A, T, h, fs, peer: Peer, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_backward_data_peer(_addr(dH, "dH", T == 0), _addr(dH_lo, "dH_lo", True), _addr(A, "A"),
                                               T, h, fs, ctypes.byref(peer), w, wn, _stream(stream)))


def mlp_tp_fc2_forward_peer_fp8(H, T, h, fs, peer: Peer, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc2_forward_peer_fp8(_addr(H, "H", T == 0, "f16"), T, h, fs, ctypes.byref(peer), w, wn,
                                             _stream(stream)))


def mlp_tp_fc1_backward_data_peer_fp8(dH, T, h, fs, peer: Peer, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_fc1_backward_data_peer_fp8(_addr(dH, "dH", T == 0, "f16"), T, h, fs, ctypes.byref(peer),
                                                   w, wn, _stream(stream)))


def mlp_tp_peer_reduce(peer: Peer, bias, T, h, out, ws, stream=None):
    w, wn = _ws(ws)
    _check(lib().mlp_tp_peer_reduce(ctypes.byref(peer), _addr(bias, "bias", True), T, h,
                                    _addr(out, "out", T == 0), w, wn, _stream(stream)))


def mlp_tp_ipc_export(ptr) -> tuple:
    """(handle bytes, offset) of the device allocation holding `ptr`."""
    handle = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_uint64(0)
    _check(lib().mlp_tp_ipc_export(_ptr(ptr), handle, ctypes.byref(off)))
    return handle.raw, int(off.value)


def mlp_tp_ipc_import(handle: bytes, offset: int) -> int:
    """Address, in this process, of the byte another process exported."""
    out = ctypes.c_void_p(0)
    buf = ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES)
    _check(lib().mlp_tp_ipc_import(buf, offset, ctypes.byref(out)))
    return int(out.value)


def mlp_tp_ipc_close(ptr: int, offset: int):
    _check(lib().mlp_tp_ipc_close(ptr, offset))


def mlp_tp_fc2_bias_grad_noalloc(dY, T, h, db, stream=None):
    """db = Σ_rows dY with no workspace (the library's static scratch)."""
    _check(lib().mlp_tp_fc2_bias_grad_noalloc(_addr(dY, "dY", T == 0), T, h, _addr(db, "db"), _stream(stream)))


def mlp_tp_check(ws, stream=None):
    """Sync the stream and read the workspace's status word (ws=None: the
    allocation-free entry point's own status word)."""
    w = None if ws is None else _ws(ws)[0]
    _check(lib().mlp_tp_check(w, _stream(stream)))


def mlp_tp_status_string(status: int) -> str:
    return lib().mlp_tp_status_string(status).decode()


def mlp_tp_last_error() -> str:
    return lib().mlp_tp_last_error().decode()


def mlp_tp_launch_count() -> int:
    return int(lib().mlp_tp_launch_count())


def mlp_tp_set_wait_budget_ns(ns: int):
    lib().mlp_tp_set_wait_budget_ns(ns)


def mlp_tp_set_debug_flags(flags: int):
    lib().mlp_tp_set_debug_flags(flags)
