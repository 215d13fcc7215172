"""The gated softmax anchor (gla_softmax_anchor) against the fp64 oracle
(oracle.softmax_anchor: QK RMSNorm, 3D RoPE, bidirectional softmax
attention, sigmoid output gate).

The kernel takes scores on the tensor cores from fp16 q_til / k_til, rounds
the softmax weights to bf16 for P V and sums those rounded weights in fp32;
the bar is the bf16 one, 2e-2 of the output RMS beyond the output's own bf16
rounding.
Small shapes and 480p are compared on every element; 720p and the 14B-width
layer on sampled heads and query rows that span the first, a middle and the
ragged last 128-token tile."""
import numpy as np
import pytest
import torch

import oracle.gla_oracle as O
from gated_bidirectional_linear_b200 import gla, workloads
from gpu_common import BF16_TOL, np64, rel_rms_bf16out

pytestmark = pytest.mark.gpu


def _draw(B, N, Hh, seed):
    x = workloads.draw(B, N, Hh, 128, "bf16", seed)
    return {n: x[n] for n in "qkvg"}


def _run(x, T, H, W, theta):
    d = {n: t.cuda() for n, t in x.items()}
    out = gla.gla_softmax_anchor(d["q"], d["k"], d["v"], d["g"], T, H, W, theta)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    return np64(out)


def _oracle(x, T, H, W, theta, b=None, h=None, queries=None):
    if b is not None:
        x = {n: t[b:b + 1, :, h:h + 1, :] for n, t in x.items()}
    a = {n: t.to(torch.float64).numpy() for n, t in x.items()}
    return O.softmax_anchor(a["q"], a["k"], a["v"], a["g"], T, H, W, theta, queries=queries)["out"]


EDGE = [
    # (B, Hh, T, H, W, theta)
    (1, 2, 2, 4, 4, 1e4),       # 32 tokens: one partial tile
    (2, 3, 1, 1, 1, 1e4),       # one token per head
    (1, 2, 1, 10, 10, 1e4),     # N = 100 < one tile
    (1, 1, 1, 8, 16, 1e4),      # N = 128: exactly one tile
    (2, 3, 5, 7, 11, 1e4),      # N = 385: three tiles and a one-token tail
    (1, 2, 3, 10, 10, 1e4),     # N = 300
    (1, 3, 7, 9, 11, 0.0),      # RoPE off
    (3, 5, 2, 16, 16, 1e4),     # N = 512: four full tiles, 15 heads
]


@pytest.mark.parametrize("case", EDGE, ids=[str(c) for c in EDGE])
def test_edge_shapes(case):
    B, Hh, T, H, W, theta = case
    x = _draw(B, T * H * W, Hh, seed=41)
    got = _run(x, T, H, W, theta)
    err = rel_rms_bf16out(got, _oracle(x, T, H, W, theta))
    print(f"anchor {case}: {err:.3e} beyond bf16 rounding")
    assert err <= BF16_TOL


def test_peaked_scores_at_the_bound():
    """q = k, RoPE off: each query's own key scores sqrt(d) log2(e) = 16.3 in
    base 2, the bound the kernel's unshifted exponentials rely on, so its
    weight 2^16.3 dominates the row."""
    B, Hh, T, H, W = 1, 2, 4, 10, 16
    x = _draw(B, T * H * W, Hh, seed=42)
    x["k"] = x["q"].clone()
    got = _run(x, T, H, W, 0.0)
    err = rel_rms_bf16out(got, _oracle(x, T, H, W, 0.0))
    print(f"anchor peaked: {err:.3e}")
    assert err <= BF16_TOL


def test_uniform_keys_read_the_mean():
    """RoPE off and one key vector for every token: all scores of a row are
    equal, so each output is sigmoid(g) * mean(v), independent of q."""
    B, Hh, T, H, W = 1, 2, 3, 9, 17
    N = T * H * W
    x = _draw(B, N, Hh, seed=43)
    x["k"] = x["k"][:, :1].expand(B, N, Hh, 128).contiguous()
    got = _run(x, T, H, W, 0.0)
    v = x["v"].to(torch.float64).numpy()
    g = x["g"].to(torch.float64).numpy()
    want = (1 / (1 + np.exp(-g))) * v.mean(axis=1, keepdims=True)
    err = rel_rms_bf16out(got, want)
    print(f"anchor uniform keys: {err:.3e}")
    assert err <= BF16_TOL


def test_480p_every_element():
    wl = workloads.WORKLOADS["480p"]
    x = _draw(wl.batch, wl.tokens, wl.heads, wl.seed)
    got = _run(x, wl.T, wl.H, wl.W, wl.rope_theta)
    err = rel_rms_bf16out(got, _oracle(x, wl.T, wl.H, wl.W, wl.rope_theta))
    print(f"anchor 480p: {err:.3e} beyond bf16 rounding")
    assert err <= BF16_TOL


def _sampled(name, heads):
    wl = workloads.WORKLOADS[name]
    x = _draw(wl.batch, wl.tokens, wl.heads, wl.seed)
    got = _run(x, wl.T, wl.H, wl.W, wl.rope_theta)
    N = wl.tokens
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([np.arange(0, 130), rng.integers(0, N, 96),
                                     np.arange(max(0, N - 130), N)]))
    worst = 0.0
    for b, h in heads:
        ref = _oracle(x, wl.T, wl.H, wl.W, wl.rope_theta, b, h, rows)
        worst = max(worst, rel_rms_bf16out(got[b:b + 1, rows, h:h + 1], ref))
    print(f"anchor {name}: sampled heads {heads}, {len(rows)} query rows each: {worst:.3e}")
    assert worst <= BF16_TOL


def test_720p_sampled_heads_and_rows():
    _sampled("720p", [(0, 0), (0, 19), (1, 7), (1, 13)])


def test_14b_sampled_heads_and_rows():
    _sampled("14b", [(0, 0), (0, 31), (0, 17)])


def test_bitwise_deterministic():
    wl = workloads.WORKLOADS["480p"]
    x = _draw(wl.batch, wl.tokens, wl.heads, wl.seed)
    a = _run(x, wl.T, wl.H, wl.W, wl.rope_theta)
    b = _run(x, wl.T, wl.H, wl.W, wl.rope_theta)
    assert np.array_equal(a, b)


def test_rejections():
    x = _draw(1, 32, 2, 44)
    d = {n: t.cuda() for n, t in x.items()}
    ws = gla.alloc_workspace(256, "cuda")
    with pytest.raises(gla.GlaError) as e:
        gla.gla_softmax_anchor(d["q"], d["k"], d["v"], d["g"], 2, 4, 4, 1e4, workspace=ws)
    assert e.value.status == gla.GLA_ERR_WORKSPACE
    y = {n: t[..., :64].contiguous() for n, t in d.items()}
    with pytest.raises(gla.GlaError) as e:
        gla.gla_softmax_anchor(y["q"], y["k"], y["v"], y["g"], 2, 4, 4, 1e4)
    assert e.value.status == gla.GLA_ERR_UNSUPPORTED
