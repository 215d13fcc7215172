"""gla_forward_noalloc: the entry point for callers that cannot allocate
device memory (its scratch is an array compiled into libgla.so).

Checked through the C ABI against gla_forward, which takes a caller-allocated
workspace, on two calls in a row each: the second call reuses the scratch the
first one left behind.  This file is collected last on purpose."""
import pytest
import torch

from gated_bidirectional_linear_b200 import gla, workloads
from gpu_common import BF16_TOL, F32_TOL, rel_floor, rel_rms, to_device

pytestmark = pytest.mark.gpu


def _both(wl, inp, tol, metric):
    d = to_device(inp)
    args = (d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W, wl.rope_theta, wl.eps)
    ref = gla.gla_forward(*args)
    for _ in range(2):
        got = gla.gla_forward_noalloc(*args)
        torch.cuda.synchronize()
        assert gla.gla_get_device_status() == gla.GLA_OK
        err = metric(got.cpu().double().numpy(), ref.cpu().double().numpy())
        assert err <= tol, err


def test_noalloc_matches_forward_fp32_tiny():
    wl = workloads.WORKLOADS["tiny"]
    _both(wl, workloads.make_inputs(wl), F32_TOL, rel_floor)


def test_noalloc_matches_forward_bf16_720p():
    wl = workloads.WORKLOADS["720p"]
    _both(wl, workloads.make_inputs(wl), BF16_TOL, rel_rms)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 4 x 64 heads of d = 128: the combined states alone exceed the array.
    d = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gla.GlaError) as e:
        gla.lib()
        st = gla.lib().gla_forward_noalloc(d.data_ptr(), d.data_ptr(), d.data_ptr(),
                                           d.data_ptr(), d.data_ptr(), 4, 64, 128, 1, 4, 32,
                                           1e4, 1e-6, gla.GLA_DTYPE_BF16, d.data_ptr(), None)
        gla._check(st, "gla_forward_noalloc")
    assert e.value.status == gla.GLA_ERR_WORKSPACE
