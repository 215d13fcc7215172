"""The oracle reproduces its stored tiny-workload result (drift guard)."""
import json
import os

import numpy as np

import oracle.gla_oracle as O
from gated_bidirectional_linear_b200 import workloads


def test_oracle_matches_stored_tiny_result():
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")) as f:
        doc = json.load(f)
    wl = workloads.WORKLOADS["tiny"]
    x = workloads.as_f64(workloads.make_inputs(wl))
    r = O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W,
                  wl.rope_theta, wl.eps)
    for key in ("out", "S", "z", "den"):
        np.testing.assert_allclose(r[key].ravel(), np.array(doc[key]), rtol=1e-12, atol=1e-12)
