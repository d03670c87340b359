"""Writes the stored expected values under tests/golden/ (calls only oracle/).

p2_example.json — the solver example on the CliffQuant project page ("Use the
solver"): weights [0.9, -0.4, 0.2, -1.1], two environment diagonals, and
QuantizerSpec(qmin=-8, qmax=7).  The page prints no output, so the expected
result is the exact-integer brute force of the definition; the weights are
first rounded to binary16 (round-to-nearest-even) and the diagonals to fp32,
because the solver's scale and inputs live on those grids.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import exact  # noqa: E402

P2_WEIGHTS = [0.9, -0.4, 0.2, -1.1]
P2_DIAGONALS = [[1.0, 0.8, 0.5, 1.2], [0.6, 1.4, 0.9, 0.7]]


def main():
    w_bits = np.array(P2_WEIGHTS, dtype=np.float64).astype(np.float16).view(np.uint16)
    d = np.array(P2_DIAGONALS, dtype=np.float64).astype(np.float32)
    r = exact.solve(w_bits, d)
    doc = {
        "source": "CliffQuant project page, section 'Use the solver' (solve_breakpoint_exact example)",
        "reading": "weights rounded to binary16 RNE, diagonals to fp32; expected values from the "
                   "exact-integer brute force over all 31,743 positive finite binary16 scales",
        "weights": P2_WEIGHTS,
        "environment_diagonals": P2_DIAGONALS,
        "qmin": -8,
        "qmax": 7,
        "w_bits": [int(x) for x in w_bits],
        "best_bits": int(r["best_bits"]),
        "best_objective": float(r["best"]),
        "best_objective_fraction": str(r["best"]),
        "runner_up_bits": int(r["runner_bits"]),
        "runner_up_objective": float(r["runner"]),
        "codes": [int(x) for x in r["codes"]],
    }
    with open(os.path.join(HERE, "p2_example.json"), "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    print(json.dumps(doc, indent=1))


if __name__ == "__main__":
    main()
