"""Write oracle_config1_head.json (a regression lock of the oracle).

Calls only the oracle and the seeded input generators.  Run from the repository
root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from doubly_stochastic_projection_b200 import inputs  # noqa: E402


def main():
    A = inputs.birkhoff_logits(4096, "normal1", 0)[:8].astype("float64")
    P_nt = oracle.newton(A, tol=1e-12, max_iter=100)
    P_sk = oracle.sinkhorn(A, iters=20)
    out = {
        "description": "oracle outputs for the first 8 matrices of the 4096-matrix N(0,1) "
                       "workload, seed 0; regression lock written by make_golden.py",
        "logits": A.tolist(),
        "newton_tol": 1e-12,
        "P_newton": P_nt.tolist(),
        "P_sinkhorn20": P_sk.tolist(),
    }
    with open(os.path.join(HERE, "oracle_config1_head.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
