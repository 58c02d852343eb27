"""Writes oracle_small.json: the oracle's outputs on tiny seeded inputs.

Calls only the oracle (and the seeded input generators).  The fixture locks
the oracle's results across compilers and machines; the pages print no
worked example with numbers, so no fixture here carries the pages' values.

    python tests/golden/make_fixtures.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from nonlinear_rnn_iteration_b200 import workloads  # noqa: E402

CASES = [
    # (workload it is shaped after, B, T, D, K, seed)
    ("linear_8x16384x1024", 1, 9, 3, 1, 101),
    ("gru_1x1024x64_k3", 1, 9, 3, 3, 102),
    ("lstm_4x32768x1024_k4", 1, 9, 2, 4, 103),
]


def main():
    out = {"generator": "tests/golden/make_fixtures.py (oracle only)", "cases": []}
    for name, B, T, D, K, seed in CASES:
        w = workloads.WORKLOADS[name].with_shape(B=B, T=T, D=D, K=K)
        x = workloads.host_inputs(w, seed=seed, with_grad=True)
        H, resid = oracle.newton(w.cell_id, x["px"], x["a"], None, K=K, nthreads=1)
        dpx, da, dh0 = oracle.adjoint(w.cell_id, x["px"], x["a"], None, H, x["dLdH"], nthreads=1)
        out["cases"].append({
            "shaped_after": name, "cell": w.cell, "B": B, "T": T, "D": D, "K": K, "seed": seed,
            "H": H.ravel().tolist(), "resid": resid.tolist(), "dLdpx": dpx.ravel().tolist(),
            "dLda": da.ravel().tolist(), "dLdh0": dh0.ravel().tolist(),
        })
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
