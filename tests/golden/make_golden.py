"""Writes tests/golden/oracle_tiny_rows.json: the fp64 oracle's outputs on the
first rows of the seeded tiny workload (T=64, H=256, V=1024, seed 0).  A
regression fixture for the oracle; it calls only oracle/ (and the seeded
input generator)."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from invariant_lm_head_gemm_b200 import workloads as wl  # noqa: E402

N_ROWS = 8


def main():
    w = wl.tiny(0)
    lp, en, ls = oracle.forward(w.hidden, w.W, w.targets, w.temperature)
    dH, dW = oracle.backward(w.hidden, w.W, w.targets, w.temperature, w.dlogp, w.dentropy)
    out = {
        "_about": "fp64 oracle on the tiny workload (seed 0), written by make_golden.py",
        "rows": N_ROWS,
        "targets": w.targets[:N_ROWS].tolist(),
        "logp": [repr(float(x)) for x in lp[:N_ROWS]],
        "entropy": [repr(float(x)) for x in en[:N_ROWS]],
        "lse": [repr(float(x)) for x in ls[:N_ROWS]],
        "dHidden_row0_first8": [repr(float(x)) for x in dH[0, :8]],
        "dW_row_target0_first8": [repr(float(x)) for x in dW[int(w.targets[0]), :8]],
        "dHidden_fro": repr(float(np.linalg.norm(dH))),
        "dW_fro": repr(float(np.linalg.norm(dW))),
    }
    with open(os.path.join(HERE, "oracle_tiny_rows.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
