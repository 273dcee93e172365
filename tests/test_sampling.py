"""The index sampler of the full-size parity tests (CPU only): it reaches
every row group, every ffn column group and both edges of every shard."""
import numpy as np

from tensor_transformer_mlp_bias_b200 import inputs
from tests.parity_util import FFN_GROUP, ROW_GROUP, sample_indices


def test_every_group_and_shard_edge_is_sampled():
    rng = np.random.default_rng(0)
    idx = sample_indices(1000, 32, rng, 250)
    assert set((idx // 32).tolist()) == set(range(32))  # the ragged last group included
    for s0 in range(0, 1000, 250):
        assert s0 in idx and s0 + 249 in idx
    assert idx.min() == 0 and idx.max() == 999


def test_large_workloads_are_covered_tile_by_tile():
    rng = np.random.default_rng(1234)
    for name in ("h4096", "8.3b-class", "175b-class"):
        wl = inputs.WORKLOADS[name]
        rows = sample_indices(wl.T, ROW_GROUP, rng)
        cols = np.unique(np.concatenate([sample_indices(wl.f, FFN_GROUP, rng, wl.f // t) for t in wl.shards]))
        # every 256-row pair tile, both of its 128-row CTA halves and all 4 lane quadrants of each
        assert set((rows // 32).tolist()) == set(range((wl.T + 31) // 32))
        # every 512-column dA tile, every 256-row dB tile and every 32-column chunk of them
        assert set((cols // 32).tolist()) == set(range((wl.f + 31) // 32))
        for t in wl.shards:
            fs = wl.f // t
            assert all(i * fs in cols and (i + 1) * fs - 1 in cols for i in range(t))
