"""Failure detection on the GPU without a fault.

Every pipeline wait in libgla is bounded: when it runs out the kernel records
a timeout in the library's device error word, stops, drains its copies and
returns, and gla_get_device_status() reports GLA_ERR_TIMEOUT.  The self-test
entry point runs that same bounded wait on an mbarrier nothing arrives on, with
a short limit, so the wait runs out for real; nothing faults, traps or hangs."""
import time

import numpy as np
import pytest
import torch

import oracle.gla_oracle as O
from gated_bidirectional_linear_b200 import gla, workloads

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_then_cleared():
    torch.cuda.set_device(0)
    assert gla.gla_get_device_status() == gla.GLA_OK          # start clean
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    gla.gla_selftest_wait_timeout(20000)                      # 20 ms
    end.record()
    t0 = time.monotonic()
    assert gla.gla_get_device_status() == gla.GLA_ERR_TIMEOUT
    assert time.monotonic() - t0 < 5.0                        # the wait did end
    assert start.elapsed_time(end) >= 19.0                    # ... after its limit
    assert gla.gla_get_device_status() == gla.GLA_OK          # reading clears it


def test_library_still_computes_after_a_timeout():
    torch.cuda.set_device(0)
    gla.gla_selftest_wait_timeout(1000)
    assert gla.gla_get_device_status() == gla.GLA_ERR_TIMEOUT
    wl = workloads.WORKLOADS["tiny"]
    inp = workloads.make_inputs(wl)
    d = {k: v.cuda() for k, v in inp.items()}
    out = gla.gla_forward(d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W)
    assert gla.gla_get_device_status() == gla.GLA_OK
    x = workloads.as_f64(inp)
    ref = O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W, 1e4, 1e-6)
    err = O.max_rel_err_rms_floor(out.cpu().double().numpy(), ref["out"])
    assert np.isfinite(err) and err <= 1e-5
