"""Write the stored oracle results under tests/golden/.

Calls only the oracle (oracle/gla_oracle.py) and the seeded input generator.
The pages print no worked numeric example of the operator, so every stored
value here is the oracle's, on the tiny workload (batch 1, 2 heads, d = 32,
2x4x4 latent grid, fp32 inputs, seed 0, theta 1e4, eps 1e-6).  The file is a
drift guard: tests/test_golden.py recomputes the oracle and compares.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from gated_bidirectional_linear_b200 import workloads  # noqa: E402
import oracle.gla_oracle as O  # noqa: E402


def main():
    wl = workloads.WORKLOADS["tiny"]
    x = workloads.as_f64(workloads.make_inputs(wl))
    r = O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W,
                  wl.rope_theta, wl.eps)
    doc = {
        "workload": "tiny: batch 1, 2 heads, d 32, grid 2x4x4, f32, seed 0, theta 1e4, eps 1e-6",
        "source": "oracle/gla_oracle.py forward(); the pages print no operator values",
        "out": r["out"].ravel().tolist(),
        "S": r["S"].ravel().tolist(),
        "z": r["z"].ravel().tolist(),
        "den": r["den"].ravel().tolist(),
    }
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()
