"""Write the stored expected values under tests/golden/ (calls oracle/ only).

Fixture ``config0_samples.json``: the 512x512 single-layer workload (seed 0,
M = 1), r in {8, 6, 4, 3, 2}; for 64 fixed output columns the fp64 oracle
value of Y = X . W_r^T.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workloads as wl  # noqa: E402


def main():
    codes, s, _ = wl.gen_weights(512, 512, wl.layer_seed(0, 0))
    _, X = wl.gen_x(1, 512, wl.layer_seed(0, 0))
    cols = list(range(0, 512, 8))
    out = {"workload": "512x512 layer, M=1, seed 0", "columns": cols, "Y": {}}
    for r in (8, 6, 4, 3, 2):
        Y = oracle.gemm(X, codes, s, r)[0]
        out["Y"][str(r)] = [float.hex(float(Y[c])) for c in cols]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "config0_samples.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)


if __name__ == "__main__":
    main()
