"""Convenience layer over the binding: allocate outputs with torch and run
the block's forward and backward through the C-ABI.  Allocation and argument
marshalling only."""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import binding


def alloc_outputs(T: int, h: int, f: int, device="cuda", with_bias_grads: bool = True,
                  mode: int = binding.ACCURATE) -> Dict[str, torch.Tensor]:
    """Outputs and saved activations; in binding.FP8 mode H is fp16 and H_lo
    holds the e4m3 residuals."""
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device=device)  # noqa: E731
    if mode == binding.FP8:
        H = torch.empty(T, f, dtype=torch.float16, device=device)
        H_lo = torch.empty(T, f, dtype=torch.float8_e4m3fn, device=device)
    else:
        H, H_lo = e(T, f), e(T, f)
    out = {"Y": e(T, h), "Z": torch.empty(T, f, dtype=torch.float32, device=device), "H": H,
           "H_lo": H_lo, "dX": e(T, h), "dA": e(h, f), "dB": e(f, h)}
    if with_bias_grads:
        out["da"] = e(f)
        out["db"] = e(h)
    return out


def forward(inp: Dict[str, torch.Tensor], t: int, out: Dict[str, torch.Tensor], ws: torch.Tensor,
            mode: int = binding.ACCURATE, stream=None) -> None:
    T, h = inp["X"].shape
    f = inp["A"].shape[1]
    binding.mlp_tp_forward(inp["X"], inp["A"], inp["a"], inp["B"], inp["b"], T, h, f, t, mode,
                           out["Y"], out["Z"], out["H"], out["H_lo"], ws, stream)


def backward(inp: Dict[str, torch.Tensor], t: int, out: Dict[str, torch.Tensor], ws: torch.Tensor,
             mode: int = binding.ACCURATE, stream=None) -> None:
    T, h = inp["X"].shape
    f = inp["A"].shape[1]
    binding.mlp_tp_backward(inp["dY"], inp["X"], inp["A"], inp["B"], out["Z"], out["H"], out["H_lo"],
                            T, h, f, t, mode, out["dX"], out["dA"], out.get("da"), out["dB"], out.get("db"),
                            ws, stream)


def forward_backward(inp: Dict[str, torch.Tensor], t: int, out: Optional[Dict[str, torch.Tensor]] = None,
                     ws: Optional[torch.Tensor] = None, mode: int = binding.ACCURATE,
                     check: bool = True) -> Dict[str, torch.Tensor]:
    """Run forward then backward on the current stream; returns the outputs.
    ``mode`` is the precision mode (binding.ACCURATE by default)."""
    T, h = inp["X"].shape
    f = inp["A"].shape[1]
    dev = inp["X"].device
    if out is None:
        out = alloc_outputs(T, h, f, dev, mode=mode)
    if ws is None:
        ws = binding.make_workspace_mode(T, h, f, t, mode, device=dev)
    forward(inp, t, out, ws, mode)
    backward(inp, t, out, ws, mode)
    if check:
        binding.mlp_tp_check(ws)
    return out
