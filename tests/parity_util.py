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


# Sampled parity at full size: one token row in every ROW_GROUP rows (the
# rows of one epilogue warp's lane quadrant: 4 per CTA, 8 per 256-row pair
# tile) and one ffn index in every FFN_GROUP columns (one epilogue chunk;
# 512-column dA tiles and 256-row dB tiles hold whole groups).
ROW_GROUP = 32
FFN_GROUP = 32


def sample_indices(n, group, rng, shard_width=None):
    """One index in every `group`-wide block of [0, n) (at a random offset;
    the last block may be ragged), the first and last index, and with
    `shard_width` the first and last index of every shard.  A whole row of Y
    or dX spans every column tile of those outputs, and a whole column of dA
    (row of dB) every row tile of it, so these indices reach every output
    tile, both CTAs of every pair, every lane quadrant and, on the ffn axis,
    every 32-column epilogue chunk and both edges of every shard."""
    idx = [min(n - 1, g + int(rng.integers(group))) for g in range(0, n, group)]
    idx += [0, n - 1]
    if shard_width is not None:
        for s0 in range(0, n, shard_width):
            idx += [s0, s0 + shard_width - 1]
    return np.unique(np.asarray(idx, dtype=np.int64))
