"""Write oracle_regression.json from the float64 oracle (calls only oracle/ and the input generator)."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import cutbce_oracle as O  # noqa: E402
from vocabulary_label_bce_b200 import workloads as W  # noqa: E402

PROBLEM = dict(T=37, V=523, D=24, K=5, dtype="bf16", seed=2024, ids="zipf", zipf_s=1.1,
               mask="random", mask_frac=0.15)


def compute():
    p = W.draw(**PROBLEM)
    out = {"problem": PROBLEM, "cases": []}
    for reduction in (O.MEAN_VALID_POSITIONS, O.SUM, O.MEAN_ELEMENTS):
        r = O.forward_backward(p.H, p.E, p.targets, p.mask, reduction=reduction, grad_loss=0.75)
        out["cases"].append({
            "reduction": reduction, "grad_loss": 0.75, "loss": r.loss, "n_valid": r.n_valid,
            "n_pairs": r.n_pairs,
            "dH_row_sums": [float(x) for x in r.dH.sum(1)],
            "dE_first_rows": [[float(x) for x in row] for row in r.dE[:3]],
            "dE_frobenius": float(np.linalg.norm(r.dE)),
        })
    return out


if __name__ == "__main__":
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression.json"), "w") as f:
        json.dump(compute(), f, indent=1)
