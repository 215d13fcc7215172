"""FP8 (OCP MX) operator inputs (gla_forward_mx) against the fp64 oracle.

The oracle decodes the same E4M3 codes and E8M0 scales (oracle.forward_mx)
and computes the operator in fp64.  Every decoded value is exact in bf16, so
the MX tensor path must also give, bit for bit, the bf16 tensor path's
output on the decoded inputs (same partitions, same arithmetic after the
decode).  Small shapes and 480p are compared on every element and on the
hidden intermediates; 720p on every head's S and z and on sampled heads'
outputs."""
import numpy as np
import pytest
import torch

import oracle.gla_oracle as O
from gated_bidirectional_linear_b200 import gla, workloads
from gpu_common import (BF16_TOL, F32_TOL, S_TOL_BF16, ZDEN_TOL, np64, rel_elem, rel_floor,
                        rel_rms, rel_rms_bf16out)

pytestmark = pytest.mark.gpu

TENSOR, SIMT, AUTO = gla.GLA_PATH_TENSOR, gla.GLA_PATH_SIMT, gla.GLA_PATH_AUTO


def _pairs(x):
    """The oracle's (codes, scales) pairs as numpy arrays."""
    return {n: (x[n].numpy(), x[n + "_scale"].numpy()) for n in "qkvg"}


def _oracle(x, T, H, W, theta=1e4, eps=1e-6, sl=None):
    p = _pairs(x)
    beta = x["beta"].to(torch.float64).numpy()
    if sl is not None:
        p = {n: (c[sl], s[sl]) for n, (c, s) in p.items()}
        beta = beta[sl[:3]]
    return O.forward_mx(p["q"], p["k"], p["v"], beta, p["g"], T, H, W, theta, eps)


def _decoded_bf16(x):
    """The decoded inputs as bf16 tensors (exact)."""
    out = {n: torch.from_numpy(O.mx_dequantize(x[n].numpy(), x[n + "_scale"].numpy())).to(
        torch.bfloat16) for n in "qkvg"}
    out["beta"] = x["beta"]
    return out


def _run(x, T, H, W, path, theta=1e4, debug=True):
    d = {k: v.cuda() for k, v in x.items()}
    r = gla.gla_forward_mx(d, T, H, W, theta, 1e-6, path=path, debug=debug)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    return {k: np64(v) for k, v in r.items()} if debug else np64(r)


def _check(got, ref, exact_arith=False):
    if exact_arith:       # CUDA-core path: fp32 arithmetic on exact decoded values
        assert rel_rms_bf16out(got["out"], ref["out"]) <= 1e-4
        assert rel_floor(got["x"], ref["x"]) <= 1e-4
        assert rel_floor(got["S"], ref["S"]) <= 1e-4
    else:
        assert rel_rms_bf16out(got["out"], ref["out"]) <= BF16_TOL
        assert rel_rms(got["x"], ref["x"]) <= BF16_TOL
        assert rel_floor(got["S"], ref["S"]) <= S_TOL_BF16
    assert rel_floor(got["z"], ref["z"]) <= ZDEN_TOL
    assert rel_elem(got["den"], ref["den"]) <= ZDEN_TOL


EDGE = [
    # (B, Hh, T, H, W, theta)
    (1, 2, 2, 4, 4, 1e4),       # 32 tokens
    (2, 3, 1, 1, 1, 1e4),       # one token per head
    (1, 5, 1, 10, 10, 1e4),     # N = 100 < one tile
    (2, 3, 5, 7, 11, 1e4),      # N = 385: a one-token tail for 96- and 128-token tiles
    (1, 2, 10, 32, 40, 1e4),    # CTAs straddle the head boundary
    (1, 3, 7, 9, 11, 0.0),      # RoPE off
]


@pytest.mark.parametrize("case", EDGE, ids=[str(c) for c in EDGE])
def test_edge_shapes_both_paths(case):
    B, Hh, T, H, W, theta = case
    x = workloads.draw_mx(B, T * H * W, Hh, 128, seed=91)
    ref = _oracle(x, T, H, W, theta)
    _check(_run(x, T, H, W, TENSOR, theta), ref)
    _check(_run(x, T, H, W, SIMT, theta), ref, exact_arith=True)


def test_mx_tensor_path_equals_bf16_path_on_decoded_inputs():
    """Bit for bit: decoding is exact, and the MX kernels do the bf16
    kernels' arithmetic on the decoded values."""
    T, H, W, B, Hh = 4, 15, 26, 1, 6
    x = workloads.draw_mx(B, T * H * W, Hh, 128, seed=17)
    got = _run(x, T, H, W, TENSOR, debug=False)
    d = {k: v.cuda() for k, v in _decoded_bf16(x).items()}
    ref = gla.gla_forward(d["q"], d["k"], d["v"], d["beta"], d["g"], T, H, W,
                          path=gla.GLA_PATH_TENSOR)
    torch.cuda.synchronize()
    assert np.array_equal(got, np64(ref))


def test_480p_all_outputs_and_intermediates():
    wl = workloads.WORKLOADS["480p"]
    x = workloads.draw_mx(wl.batch, wl.tokens, wl.heads, wl.head_dim, wl.seed)
    ref = _oracle(x, wl.T, wl.H, wl.W)
    got = _run(x, wl.T, wl.H, wl.W, TENSOR)
    print(f"MX 480p: out {rel_rms(got['out'], ref['out']):.3e} of the RMS "
          f"({rel_rms_bf16out(got['out'], ref['out']):.3e} beyond bf16 rounding), x "
          f"{rel_rms(got['x'], ref['x']):.3e}, S {rel_floor(got['S'], ref['S']):.3e}, z "
          f"{rel_floor(got['z'], ref['z']):.3e}, den {rel_elem(got['den'], ref['den']):.3e}")
    _check(got, ref)


def test_720p_every_state_sampled_outputs():
    wl = workloads.WORKLOADS["720p"]
    x = workloads.draw_mx(wl.batch, wl.tokens, wl.heads, wl.head_dim, wl.seed)
    got = _run(x, wl.T, wl.H, wl.W, AUTO)
    worst = dict(S=0.0, z=0.0, out=0.0)
    for b in range(wl.batch):
        for h in range(wl.heads):
            sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
            ref = _oracle(x, wl.T, wl.H, wl.W, sl=sl)
            worst["S"] = max(worst["S"], rel_floor(got["S"][b, h], ref["S"][0, 0]))
            worst["z"] = max(worst["z"], rel_floor(got["z"][b, h], ref["z"][0, 0]))
            if (b, h) in [(0, 0), (0, 19), (1, 7), (1, 13)]:
                worst["out"] = max(worst["out"], rel_rms_bf16out(got["out"][sl], ref["out"]))
    print(f"MX 720p: every head S {worst['S']:.3e}, z {worst['z']:.3e}; sampled outputs "
          f"{worst['out']:.3e} beyond bf16 rounding")
    assert worst["S"] <= S_TOL_BF16 and worst["z"] <= ZDEN_TOL and worst["out"] <= BF16_TOL


def test_bitwise_deterministic():
    wl = workloads.WORKLOADS["480p"]
    x = workloads.draw_mx(wl.batch, wl.tokens, wl.heads, wl.head_dim, wl.seed)
    a = _run(x, wl.T, wl.H, wl.W, AUTO, debug=False)
    b = _run(x, wl.T, wl.H, wl.W, AUTO, debug=False)
    assert np.array_equal(a, b)
