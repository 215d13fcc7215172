"""Token-level causal variant (gla_causal_step) against the fp64 oracle.

Small shapes are compared on every output and on the exported denominator and
pre-norm read-out (oracle.causal_forward, running sums); the pre-norm read-out
is measured against each token's own RMS, since its scale varies from token
to token (an early token averages a few values, a late one many); the 480p shape on
every token of sampled heads; the full 720p shape on sampled tokens of sampled
heads, each recomputed by the oracle from its own prefix
(oracle.causal_forward_at).  The state after the call is compared with the
oracle's full-sequence state on every head.  Streaming (a sequence split over
two calls), determinism and the CUDA-core / tensor agreement are checked too."""
import numpy as np
import pytest
import torch

import oracle.gla_oracle as O
from gated_bidirectional_linear_b200 import gla, workloads
from gpu_common import (BF16_TOL, F32_TOL, S_TOL_BF16, ZDEN_TOL, head_slice, np64, rel_elem,
                        rel_floor, rel_rms, rel_rms_bf16out, rel_row_rms, to_device)

pytestmark = pytest.mark.gpu

TENSOR, SIMT, AUTO = gla.GLA_PATH_TENSOR, gla.GLA_PATH_SIMT, gla.GLA_PATH_AUTO


def _run(inp, T, H, W, theta, eps, path, t0=0, state=None, z=None):
    d = to_device(inp)
    B, N, Hh, hd = d["q"].shape
    S = torch.zeros(B, Hh, hd, hd, device="cuda") if state is None else state.clone().cuda()
    zz = torch.zeros(B, Hh, hd, device="cuda") if z is None else z.clone().cuda()
    den = torch.empty(B, N, Hh, device="cuda")
    x = torch.empty(B, N, Hh, hd, device="cuda")
    out = gla.gla_causal_step(S, zz, d["q"], d["k"], d["v"], d["beta"], d["g"], T, H, W, t0,
                              theta, eps, path=path, den_out=den, x_out=x)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    return dict(out=np64(out), den=np64(den), x=np64(x), S=np64(S), z=np64(zz))


def _oracle(inp, T, H, W, theta, eps, t0=0):
    x = inp if isinstance(inp["q"], np.ndarray) else workloads.as_f64(inp)
    r = O.causal_forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W, theta, eps, t0)
    f = O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W, theta, eps, t0)
    r.update(S=f["S"], z=f["z"])       # the state after the last token
    return r


def _check(got, ref, dtype):
    if dtype == "f32":
        assert rel_floor(got["out"], ref["out"]) <= F32_TOL
        assert rel_floor(got["x"], ref["x"]) <= F32_TOL
        assert rel_floor(got["S"], ref["S"]) <= F32_TOL
    else:
        assert rel_rms_bf16out(got["out"], ref["out"]) <= BF16_TOL
        assert rel_row_rms(got["x"], ref["x"]) <= BF16_TOL
        assert rel_floor(got["S"], ref["S"]) <= S_TOL_BF16
    assert rel_floor(got["z"], ref["z"]) <= ZDEN_TOL
    assert rel_elem(got["den"], ref["den"]) <= ZDEN_TOL
    assert np.all(got["den"] >= 1e-6 * (1 - 1e-6))


def test_tiny_fp32_all_outputs():
    wl = workloads.WORKLOADS["tiny"]
    inp = workloads.make_inputs(wl)
    got = _run(inp, wl.T, wl.H, wl.W, wl.rope_theta, wl.eps, AUTO)
    _check(got, _oracle(inp, wl.T, wl.H, wl.W, wl.rope_theta, wl.eps), "f32")


EDGE = [
    # (B, Hh, d, T, H, W, dtype, theta)
    (2, 3, 128, 1, 1, 1, "bf16", 1e4),        # one token per head
    (1, 5, 128, 1, 10, 10, "bf16", 1e4),      # N = 100: one chunk and four rows
    (2, 3, 128, 1, 1, 193, "bf16", 1e4),      # two chunks and a one-token tail
    (1, 2, 128, 10, 32, 40, "bf16", 1e4),     # CTAs straddle the head boundary
    (1, 3, 128, 7, 9, 11, "bf16", 0.0),       # RoPE off
    (1, 4, 64, 3, 5, 7, "bf16", 1e4),         # d = 64 (CUDA-core path)
    (2, 3, 64, 3, 5, 7, "f32", 1e4),          # fp32, d = 64
    (1, 2, 128, 2, 3, 33, "f32", 1e4),        # fp32, d = 128
]


@pytest.mark.parametrize("case", EDGE, ids=[str(c) for c in EDGE])
def test_edge_shapes(case):
    B, Hh, d, T, H, W, dt, theta = case
    inp = workloads.draw(B, T * H * W, Hh, d, dt, seed=321)
    ref = _oracle(inp, T, H, W, theta, 1e-6)
    paths = [AUTO] + ([SIMT] if (dt == "bf16" and d == 128) else [])
    for path in paths:
        _check(_run(inp, T, H, W, theta, 1e-6, path), ref, dt)


@pytest.fixture(scope="module")
def c480():
    wl = workloads.WORKLOADS["480p"]
    return wl, workloads.make_inputs(wl)


@pytest.mark.parametrize("path", [TENSOR, SIMT], ids=["tensor", "simt"])
def test_480p_sampled_heads_every_token(c480, path):
    wl, inp = c480
    got = _run(inp, wl.T, wl.H, wl.W, wl.rope_theta, wl.eps, path)
    worst = dict(out=0.0, raw=0.0, x=0.0, den=0.0)
    for b, h in [(0, 0), (0, 9), (0, 19)]:
        ref = _oracle(head_slice(inp, b, h), wl.T, wl.H, wl.W, wl.rope_theta, wl.eps)
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        worst["out"] = max(worst["out"], rel_rms_bf16out(got["out"][sl], ref["out"]))
        worst["raw"] = max(worst["raw"], rel_rms(got["out"][sl], ref["out"]))
        worst["x"] = max(worst["x"], rel_row_rms(got["x"][sl], ref["x"]))
        worst["den"] = max(worst["den"], rel_elem(got["den"][sl], ref["den"]))
    # the state after the call, every head
    x = workloads.as_f64(inp)
    full = O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W,
                     wl.rope_theta, wl.eps)
    eS = rel_floor(got["S"], full["S"])
    ez = rel_floor(got["z"], full["z"])
    print(f"causal 480p path {path}: out {worst['raw']:.3e} of the RMS ({worst['out']:.3e} "
          f"beyond bf16 rounding), x {worst['x']:.3e}, den {worst['den']:.3e}, end S {eS:.3e}, "
          f"end z {ez:.3e}")
    assert worst["out"] <= BF16_TOL and worst["x"] <= BF16_TOL
    assert worst["den"] <= ZDEN_TOL
    assert eS <= S_TOL_BF16 and ez <= ZDEN_TOL


def test_720p_sampled_tokens():
    """The benchmarked shape on the tensor path (gla_causal_step as the
    benchmark calls it): 12 tokens of 4 heads, chosen at chunk and CTA edges
    and spread over the sequence, each recomputed from its own prefix."""
    wl = workloads.WORKLOADS["720p"]
    inp = workloads.make_inputs(wl)
    d = to_device(inp)
    B, N, Hh, hd = d["q"].shape
    S = torch.zeros(B, Hh, hd, hd, device="cuda")
    z = torch.zeros(B, Hh, hd, device="cuda")
    out = gla.gla_causal_step(S, z, d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    out = np64(out)
    toks = [0, 1, 95, 96, 97, 191, 4000, 7777, 9983, 12000, N - 2, N - 1]
    worst, worst_raw = 0.0, 0.0
    for b, h in [(0, 0), (0, 13), (1, 6), (1, 19)]:
        x = head_slice(inp, b, h)
        ref = O.causal_forward_at(x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W,
                                  wl.rope_theta, wl.eps, toks)
        got = out[b:b + 1, toks, h:h + 1]
        worst = max(worst, rel_rms_bf16out(got, ref["out"]))
        worst_raw = max(worst_raw, rel_rms(got, ref["out"]))
        assert rel_floor(np64(S[b, h]), ref["S_end"][0, 0]) <= S_TOL_BF16
        assert rel_floor(np64(z[b, h]), ref["z_end"][0, 0]) <= ZDEN_TOL
    print(f"causal 720p sampled tokens: out {worst_raw:.3e} of the RMS ({worst:.3e} beyond bf16 "
          f"rounding)")
    assert worst <= BF16_TOL


def test_streaming_two_calls_equal_one():
    """A sequence split over two calls (the second from the first's state,
    its frames offset by t0) gives the one-call outputs within rounding, and
    the same end state."""
    T, H, W, B, HH = 6, 8, 20, 1, 4
    inp = workloads.draw(B, T * H * W, HH, 128, "bf16", seed=77)
    one = _run(inp, T, H, W, 1e4, 1e-6, AUTO)
    L = (T // 2) * H * W
    first = {k: v[:, :L].contiguous() for k, v in inp.items()}
    second = {k: v[:, L:].contiguous() for k, v in inp.items()}
    a = _run(first, T // 2, H, W, 1e4, 1e-6, AUTO)
    b = _run(second, T // 2, H, W, 1e4, 1e-6, AUTO, t0=T // 2, state=torch.from_numpy(a["S"]).float(),
             z=torch.from_numpy(a["z"]).float())
    both = np.concatenate([a["out"], b["out"]], axis=1)
    assert rel_rms(both, one["out"]) <= BF16_TOL
    # the same fp32 sums grouped differently (two partitions of the tokens)
    assert rel_floor(b["S"], one["S"]) <= 1e-4
    x = workloads.as_f64(inp)
    ref = O.causal_forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W, 1e4, 1e-6)
    assert rel_rms_bf16out(both, ref["out"]) <= BF16_TOL


def test_bitwise_deterministic():
    wl = workloads.WORKLOADS["480p"]
    d = to_device(workloads.make_inputs(wl))
    a = gla.gla_causal_forward(d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W)
    b = gla.gla_causal_forward(d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_tensor_and_cuda_core_paths_agree(c480):
    wl, inp = c480
    a = _run(inp, wl.T, wl.H, wl.W, wl.rope_theta, wl.eps, TENSOR)
    b = _run(inp, wl.T, wl.H, wl.W, wl.rope_theta, wl.eps, SIMT)
    assert rel_row_rms(a["x"], b["x"]) <= BF16_TOL
    assert rel_elem(a["den"], b["den"]) <= ZDEN_TOL


def test_host_entry_matches_device_entry():
    """gla_causal_step_host (host inputs and output, device-resident state)
    gives gla_causal_step's output and state bit for bit, over two calls."""
    T, H, W, B, HH = 4, 6, 10, 2, 3
    L = (T // 2) * H * W
    inp = workloads.draw(B, T * H * W, HH, 128, "bf16", seed=55)
    S_d = torch.zeros(B, HH, 128, 128, device="cuda")
    z_d = torch.zeros(B, HH, 128, device="cuda")
    S_h, z_h = S_d.clone(), z_d.clone()
    for i in range(2):
        part = {k: v[:, i * L:(i + 1) * L].contiguous() for k, v in inp.items()}
        d = to_device(part)
        o_d = gla.gla_causal_step(S_d, z_d, d["q"], d["k"], d["v"], d["beta"], d["g"], T // 2, H,
                                  W, i * (T // 2))
        p = {k: v.pin_memory() for k, v in part.items()}
        o_h = torch.empty_like(p["q"]).pin_memory()
        gla.gla_causal_step_host(S_h, z_h, p["q"], p["k"], p["v"], p["beta"], p["g"], T // 2, H,
                                 W, i * (T // 2), out=o_h)
        torch.cuda.synchronize()
        assert gla.gla_get_device_status() == gla.GLA_OK
        assert torch.equal(o_h, o_d.cpu())
    assert torch.equal(S_h, S_d) and torch.equal(z_h, z_d)
