"""Write tests/golden/tiny_flce.json from the float64 oracle alone.

The pages print no worked FLCE example, so every stored value here comes from
oracle/ on the seeded tiny workload (BT=512, H=256, V=4096, fp32, 5% ignored,
seed 0). Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from linear_cross_entropy_04_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def main():
    w = WORKLOADS["tiny"]
    d = make_inputs(w)
    out = {"workload": "tiny FLCE: BT=512 H=256 V=4096 fp32, W~N(0,0.02), uniform targets, 5% ignore, seed 0",
           "source": "oracle.flce (float64)"}
    for red in ("mean", "sum"):
        r = oracle.flce(d["X"], d["W"], d["target"], reduction=red)
        out[red] = {
            "loss": r["loss"],
            "n_valid": r["n_valid"],
            "row_loss_first16": r["row_loss"][:16].tolist(),
            "grad_X_row0_first8": r["grad_X"][0, :8].tolist(),
            "grad_W_rows0to3_first8": r["grad_W"][:4, :8].tolist(),
            "grad_X_abs_sum": float(np.abs(r["grad_X"]).sum()),
            "grad_W_abs_sum": float(np.abs(r["grad_W"]).sum()),
        }
    with open(os.path.join(HERE, "tiny_flce.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
