"""Writes tests/golden/tiny_seed0.json from the fp64 oracle alone.

The pages print no worked numeric example of the MLP block, so this fixture
is a regression record of the oracle on the tiny workload (T=64, h=256,
f=1024, seed 0): it guards the oracle and the seeded generator against silent
drift.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import mlp_oracle  # noqa: E402
from tensor_transformer_mlp_bias_b200 import inputs  # noqa: E402


def main():
    inp = inputs.make_inputs(inputs.WORKLOADS["tiny"])
    out = mlp_oracle.full(inp)
    rec = {
        "workload": "tiny T=64 h=256 f=1024 seed=0",
        "source": "oracle/mlp_oracle.py full(); regression record, not a page value",
        "Y[0,:8]": out["Y"][0, :8].tolist(),
        "Y[63,-8:]": out["Y"][63, -8:].tolist(),
        "Z[1,:8]": out["Z"][1, :8].tolist(),
        "H[1,:8]": out["H"][1, :8].tolist(),
        "dX[2,:8]": out["dX"][2, :8].tolist(),
        "dA[3,:8]": out["dA"][3, :8].tolist(),
        "da[:8]": out["da"][:8].tolist(),
        "dB[4,:8]": out["dB"][4, :8].tolist(),
        "db[:8]": out["db"][:8].tolist(),
    }
    with open(os.path.join(HERE, "tiny_seed0.json"), "w") as fh:
        json.dump(rec, fh, indent=1)
        fh.write("\n")


if __name__ == "__main__":
    main()
