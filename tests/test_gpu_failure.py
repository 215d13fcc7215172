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


def test_state_pipeline_abort_path_then_recovery():
    """The state kernel's own abort path: CTA 0's producer withholds one
    arrival, the transform warps' wait runs out after 2 ms, and every role
    leaves, drains its copies and MMAs and frees TMEM; the call ends, the
    status reads GLA_ERR_TIMEOUT once, and the next call matches the oracle."""
    torch.cuda.set_device(0)
    assert gla.gla_get_device_status() == gla.GLA_OK
    T, H, W, B, HH = 2, 6, 16, 1, 3
    inp = workloads.draw(B, T * H * W, HH, 128, "bf16", seed=61)
    d = {k: v.cuda() for k, v in inp.items()}
    t0 = time.monotonic()
    gla.gla_selftest_pipeline_stall(d["q"], d["k"], d["v"], d["beta"], d["g"], T, H, W, 2000)
    assert gla.gla_get_device_status() == gla.GLA_ERR_TIMEOUT
    assert time.monotonic() - t0 < 10.0
    assert gla.gla_get_device_status() == gla.GLA_OK
    out = gla.gla_forward(d["q"], d["k"], d["v"], d["beta"], d["g"], T, H, W)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    x = workloads.as_f64(inp)
    ref = O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W, 1e4, 1e-6)
    assert O.bf16_out_err_over_rms(out.cpu().double().numpy(), ref["out"]) <= 2e-2
