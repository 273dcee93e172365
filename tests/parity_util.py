"""Helpers shared by the GPU parity tests."""
from __future__ import annotations

import numpy as np
import torch

# Elementwise bar for forward and gradients: max |gpu − oracle| ≤ 1e-2·(|oracle| + 1).
RTOL = 1e-2


def to_gpu(inp):
    return {k: v.cuda() for k, v in inp.items()}


def to_np(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.float64).numpy()


def worst_ratio(gpu, ref) -> float:
    """max over elements of |gpu − ref| / (RTOL·(|ref| + 1)); ≤ 1 passes."""
    g = to_np(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if g.size == 0:
        return 0.0
    if not np.all(np.isfinite(g)):
        return float("inf")
    return float(np.max(np.abs(g - r) / (RTOL * (np.abs(r) + 1.0))))


def assert_close(name, gpu, ref):
    w = worst_ratio(gpu, ref)
    assert w <= 1.0, f"{name}: worst |gpu-oracle| / (1e-2(|oracle|+1)) = {w:.3f}"
    return w


def bits(x: torch.Tensor) -> torch.Tensor:
    return x.contiguous().view(torch.int16)
