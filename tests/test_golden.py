"""Golden regression record of the oracle on the tiny workload."""
import json
import os

import numpy as np

from oracle import mlp_oracle
from tensor_transformer_mlp_bias_b200 import inputs

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_reproduces_golden_record():
    with open(os.path.join(HERE, "tiny_seed0.json")) as fh:
        rec = json.load(fh)
    out = mlp_oracle.full(inputs.make_inputs(inputs.WORKLOADS["tiny"]))
    got = {
        "Y[0,:8]": out["Y"][0, :8], "Y[63,-8:]": out["Y"][63, -8:],
        "Z[1,:8]": out["Z"][1, :8], "H[1,:8]": out["H"][1, :8],
        "dX[2,:8]": out["dX"][2, :8], "dA[3,:8]": out["dA"][3, :8],
        "da[:8]": out["da"][:8], "dB[4,:8]": out["dB"][4, :8], "db[:8]": out["db"][:8],
    }
    for k, v in got.items():
        np.testing.assert_allclose(v, np.array(rec[k]), rtol=1e-12, atol=1e-12, err_msg=k)


def test_generator_is_bf16_and_seeded():
    wl = inputs.WORKLOADS["tiny"]
    i1 = inputs.make_inputs(wl)
    i2 = inputs.make_inputs(wl)
    for k in i1:
        assert i1[k].dtype.is_floating_point and str(i1[k].dtype) == "torch.bfloat16"
        assert bool((i1[k].view(-1).view(dtype=__import__("torch").int16)
                     == i2[k].view(-1).view(dtype=__import__("torch").int16)).all())
    assert tuple(i1["X"].shape) == (64, 256) and tuple(i1["A"].shape) == (256, 1024)
    assert tuple(i1["B"].shape) == (1024, 256) and tuple(i1["dY"].shape) == (64, 256)
    # distribution sanity: weights ~N(0, 0.02)
    assert abs(float(i1["A"].float().std()) - 0.02) < 0.001
