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


def _scratch_bytes():
    """GLA_NOALLOC_SCRATCH_BYTES as include/gla.h defines it."""
    import os
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "include", "gla.h")
    m = re.search(r"#define GLA_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", open(hdr).read())
    assert m, "GLA_NOALLOC_SCRATCH_BYTES not found in gla.h"
    return int(m.group(1)) << int(m.group(2))


def test_noalloc_matches_forward_fp32_720p_simt():
    """fp32 inputs at the 720p shape run on the CUDA-core path, whose scratch
    (no fp16 image, no read-out table) fits the array."""
    wl = workloads.WORKLOADS["720p"]
    inp = workloads.draw(wl.batch, wl.tokens, wl.heads, wl.head_dim, "f32", wl.seed)
    _both(wl, inp, F32_TOL, rel_floor)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # Enough heads that the combined fp32 states alone (heads x d x d x 4
    # bytes, one part of the scratch) take twice the array; one token each.
    # Every buffer passed has the problem's real size, and the host checks
    # from the same formula that the problem is beyond the array.
    cap, d = _scratch_bytes(), 128
    heads = 2 * cap // (d * d * 4) + 32
    assert heads * d * d * 4 > 2 * cap
    x = workloads.draw(1, 1, heads, d, "bf16", seed=3)
    x = to_device(x)
    out = torch.empty_like(x["q"])
    with pytest.raises(gla.GlaError) as e:
        gla.gla_forward_noalloc(x["q"], x["k"], x["v"], x["beta"], x["g"], 1, 1, 1, out=out)
    assert e.value.status == gla.GLA_ERR_WORKSPACE
