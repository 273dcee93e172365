"""Seeded synthetic inputs and the named workload shapes.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests.  It holds no arithmetic of the MLP block: it only draws Gaussian
tensors from a seeded torch CPU generator and rounds them to bf16, so both
sides see bit-identical inputs.

Workloads (tokens T, hidden h, ffn f, shard counts t) are the tensor-parallel
MLP shapes of the Megatron-LM line of work: a tiny block, a GPT-2-medium
block, an 8.3B-class layer (the 2019 paper's largest model, "Megatron-LM 深度解读报告"
§四 4.1 table), an h=4096 layer and a 175B-class layer.

Draw order is fixed: X, A, a, B, b, dY, each as fp32 randn * std, then
round-to-nearest-even to bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens (rows of X)
    h: int            # hidden size
    f: int            # ffn size (columns of A, rows of B)
    shards: Tuple[int, ...]   # tensor-parallel shard counts t to run
    w_std: float      # std of A and B
    bias_std: float = 0.02
    x_std: float = 1.0
    dy_std: float = 1.0
    seed: int = 0

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of one forward+backward: six GEMMs of 2*T*h*f."""
        return 12 * self.T * self.h * self.f


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 64, 256, 1024, (2,), 0.02),
    "gpt2-medium": Workload("gpt2-medium", 8 * 1024, 1024, 4096, (1, 2, 4, 8), 0.02),
    "8.3b-class": Workload("8.3b-class", 16 * 1024, 3072, 12288, (8,), 0.02),
    # weights ~ N(0, 0.02/sqrt(2*layers)) with 32 layers
    "h4096": Workload("h4096", 8 * 512, 4096, 16384, (1, 4, 8), 0.02 / math.sqrt(2 * 32)),
    "175b-class": Workload("175b-class", 4 * 2048, 12288, 49152, (8,), 0.006),
}

HEADLINE = "h4096"


def make_inputs(wl: Workload, seed: int | None = None, T: int | None = None):
    """Return dict of bf16 CPU tensors X[T,h], A[h,f], a[f], B[f,h], b[h], dY[T,h].

    ``T`` overrides the token count (same distributions); ``seed`` overrides
    the workload's seed.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed if seed is None else seed)
    T = wl.T if T is None else T

    def draw(shape, std):
        return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)

    X = draw((T, wl.h), wl.x_std)
    A = draw((wl.h, wl.f), wl.w_std)
    a = draw((wl.f,), wl.bias_std)
    B = draw((wl.f, wl.h), wl.w_std)
    b = draw((wl.h,), wl.bias_std)
    dY = draw((T, wl.h), wl.dy_std)
    return {"X": X, "A": A, "a": a, "B": B, "b": b, "dY": dY}


def make_custom(T: int, h: int, f: int, w_std: float = 0.02, bias_std: float = 0.02,
                seed: int = 0):
    """Inputs for an arbitrary shape (edge-case and ragged tests)."""
    wl = Workload("custom", T, h, f, (1,), w_std, bias_std, seed=seed)
    return make_inputs(wl)
