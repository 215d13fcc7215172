"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each check_* function raises AssertionError when the oracle disagrees with a
closed form, a brute-force sum, a textbook special case or an invariant that
the pages and the mathematics fix.  The checks look up every oracle function
through the module object at call time, so tests/test_oracle_mutants.py can
plant a mistake in the oracle and verify that at least one check fails.

Sources are cited by page title and section:
[GBLA] SANA-Video 2.0 summary (paper.rainbus.top), prerequisites, "Gated
       Bilinear Linear Attention" (read-out formula).
[LA]   same page, prerequisites, "Linear Attention" (state S = sum v (beta k)^T).
[V1]   SANA-Video notes (papernotes.org), key design 1 (RoPE(ReLU(x)),
       numerator only, positive denominator).
[BLK]  same notes, key design 2 (block-causal running sums).
"""
import math

import numpy as np

import oracle.gla_oracle as O
from gated_bidirectional_linear_b200 import workloads

EPS_N = 1e-6  # RMSNorm epsilon of the spec


def _close(got, want, tol, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.max(np.abs(got - want) / np.maximum(np.abs(want), 1e-300 + np.abs(want).max()))
    assert err <= tol, f"{what}: rel err {err:.3e} > {tol:.1e}\n got={got}\nwant={want}"


def _rms_scale(x):
    return 1.0 / math.sqrt(sum(e * e for e in x) / len(x) + EPS_N)


def _inputs_f64(wl):
    return workloads.as_f64(workloads.make_inputs(wl))


# ---------------------------------------------------------------- closed forms

def check_single_token_closed_form():
    """N = 1 at position 0 (no rotation).  S = v (beta k_pls)^T, so
    pre = v beta c / (c + eps) with c = k_pls . q_pls ([LA], [GBLA]).
    q = (1,1,1,1): q_pls = q / sqrt(1 + e_n).  k = (2,-2,2,-2): ReLU keeps
    (2,0,2,0) / sqrt(4 + e_n).  c = 4 / (sqrt(4+e_n) sqrt(1+e_n))."""
    eps = 1e-3
    q = np.array([1.0, 1.0, 1.0, 1.0])
    k = np.array([2.0, -2.0, 2.0, -2.0])
    v = np.array([1.0, 2.0, 3.0, 4.0])
    beta = 0.5
    g = np.array([0.0, math.log(3.0), -math.log(3.0), 0.0])     # sigma = .5 .75 .25 .5
    c = 4.0 / (math.sqrt(4.0 + EPS_N) * math.sqrt(1.0 + EPS_N))
    s = beta * c / (c + eps)
    x = [0.5 * 1.0 * s, 0.75 * 2.0 * s, 0.25 * 3.0 * s, 0.5 * 4.0 * s]
    out_want = [e * _rms_scale(x) for e in x]
    shp = (1, 1, 1, 4)
    r = O.forward(q.reshape(shp), k.reshape(shp), v.reshape(shp), np.full((1, 1, 1), beta),
                  g.reshape(shp), 1, 1, 1, 10000.0, eps)
    _close(r["x"].ravel(), x, 1e-12, "N=1 gated read-out")
    _close(r["out"].ravel(), out_want, 1e-12, "N=1 output")
    _close(r["den"].ravel(), [c + eps], 1e-12, "N=1 denominator")


def _two_token_case():
    """Two tokens on the time axis (T=2, H=W=1), d = 2: one rotation pair with
    frequency theta^0 = 1, so token 1 is rotated by exactly 1 rad.

    k0 = (1, 0):  k_pls0 = (a, 0),            a = 1/sqrt(0.5 + e_n)
    k1 = (-1, 1): k_pls1 = (0, b),            b = 1/sqrt(1 + e_n)
                  k_til1 = (-b sin1, b cos1)  (rotation after the ReLU)
    q0 = (0, 2):  q_pls0 = q_til0 = (0, c2),  c2 = 2/sqrt(2 + e_n)
    q1 = (3, 1):  q_pls1 = (3e, e),           e = 1/sqrt(5 + e_n)
                  q_til1 = (3e cos1 - e sin1, 3e sin1 + e cos1)
    Dot products: k_til0.q_til0 = 0, k_til1.q_til0 = b c2 cos1,
                  k_til0.q_til1 = a e (3 cos1 - sin1), k_til1.q_til1 = b e.
    Denominators (no rotation): den0 = b c2 + eps, den1 = 3 a e + b e + eps.
    """
    eps = 1e-2
    s1, c1 = math.sin(1.0), math.cos(1.0)
    a = 1.0 / math.sqrt(0.5 + EPS_N)
    b = 1.0 / math.sqrt(1.0 + EPS_N)
    c2 = 2.0 / math.sqrt(2.0 + EPS_N)
    e = 1.0 / math.sqrt(5.0 + EPS_N)
    v0, v1 = np.array([1.0, -1.0]), np.array([2.0, 0.5])
    be0, be1 = 0.5, 0.25
    pre0 = v1 * be1 * (b * c2 * c1) / (b * c2 + eps)
    pre1 = (v0 * be0 * (a * e * (3 * c1 - s1)) + v1 * be1 * (b * e)) / (3 * a * e + b * e + eps)
    sig0 = np.array([0.5, 0.75])                      # g0 = (0, ln 3)
    sig1 = np.array([0.25, 0.5])                      # g1 = (-ln 3, 0)
    x0, x1 = sig0 * pre0, sig1 * pre1
    want = dict(
        den=[b * c2 + eps, 3 * a * e + b * e + eps],
        pre=np.stack([pre0, pre1]),
        out=np.stack([x0 * _rms_scale(x0), x1 * _rms_scale(x1)]),
    )
    q = np.array([[0.0, 2.0], [3.0, 1.0]]).reshape(1, 2, 1, 2)
    k = np.array([[1.0, 0.0], [-1.0, 1.0]]).reshape(1, 2, 1, 2)
    v = np.stack([v0, v1]).reshape(1, 2, 1, 2)
    beta = np.array([be0, be1]).reshape(1, 2, 1)
    g = np.array([[0.0, math.log(3.0)], [-math.log(3.0), 0.0]]).reshape(1, 2, 1, 2)
    return (q, k, v, beta, g, 2, 1, 1, 10000.0, eps), want


def check_two_token_closed_form():
    args, want = _two_token_case()
    r = O.forward(*args)
    _close(r["den"].ravel(), want["den"], 1e-12, "N=2 denominators")
    _close(r["pre"].reshape(2, 2), want["pre"], 1e-12, "N=2 pre-gate read-out")
    _close(r["out"].reshape(2, 2), want["out"], 1e-12, "N=2 output")


def check_two_token_bruteforce_closed_form():
    args, want = _two_token_case()
    r = O.forward_bruteforce(*args)
    _close(r["pre"].reshape(2, 2), want["pre"], 1e-12, "N=2 brute force")
    _close(r["out"].reshape(2, 2), want["out"], 1e-12, "N=2 brute-force output")


# ------------------------------------------------------------ RoPE (the spec)

def check_rope_split():
    assert O.rope_pair_split(128) == (22, 21, 21)
    assert O.rope_pair_split(32) == (6, 5, 5)
    assert O.rope_pair_split(6) == (1, 1, 1)
    assert O.rope_pair_split(2) == (1, 0, 0)


def check_rope_axis_order():
    """d = 6: pair 0 turns with t, pair 1 with h, pair 2 with w, each at
    frequency 1.  Token (t,h,w) = (1,2,3) of a 2x3x4 grid is n = 23; the unit
    vector (1,0,1,0,1,0) goes to (cos1, sin1, cos2, sin2, cos3, sin3)."""
    ang = O.rope_angles(6, 2, 3, 4, 10000.0)
    x = np.zeros((1, 24, 1, 6))
    x[..., 0::2] = 1.0
    y = O.rope_rotate(x, ang)[0, 23, 0]
    want = [math.cos(1), math.sin(1), math.cos(2), math.sin(2), math.cos(3), math.sin(3)]
    _close(y, want, 1e-15, "RoPE axis order")


def check_rope_frequencies():
    """d = 12, theta = 1e4: two pairs per axis with frequencies 1 and
    theta^(-1/2) = 0.01.  Token (t,h,w) = (0,0,3) turns only the w pairs
    (channels 8..11) by 3 and 0.03 rad; (x0, x1) = (0, 1) -> (-sin, cos)."""
    ang = O.rope_angles(12, 1, 1, 4, 10000.0)
    x = np.zeros((1, 4, 1, 12))
    x[..., 1::2] = 1.0
    y = O.rope_rotate(x, ang)[0, 3, 0]
    want = [0, 1, 0, 1, 0, 1, 0, 1, -math.sin(3), math.cos(3), -math.sin(0.03), math.cos(0.03)]
    assert np.max(np.abs(y - np.array(want))) < 1e-15, f"RoPE frequencies: {y}"


def check_rope_complex_form():
    """Rotating pair (x0, x1) equals multiplying x0 + i x1 by exp(i angle)."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 40, 2, 32))
    ang = O.rope_angles(32, 2, 4, 5, 500.0, t0=3)
    y = O.rope_rotate(x, ang)
    zc = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * ang)[None, :, None, :]
    assert np.max(np.abs(y[..., 0::2] - zc.real)) < 1e-13
    assert np.max(np.abs(y[..., 1::2] - zc.imag)) < 1e-13


# ------------------------------------------------- brute force and invariants

def check_factorised_equals_bruteforce():
    """Tiny workload (1x2 heads, d=32, 2x4x4 grid, seed 0): the S/z form and
    the O(N^2) pair sum agree to fp64 rounding, before and after gate/norm."""
    wl = workloads.WORKLOADS["tiny"]
    x = _inputs_f64(wl)
    args = (x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W, wl.rope_theta, wl.eps)
    f = O.forward(*args)
    bf = O.forward_bruteforce(*args)
    _close(f["pre"], bf["pre"], 1e-12, "factorised vs brute force (pre)")
    _close(f["out"], bf["out"], 1e-12, "factorised vs brute force (out)")


def check_bruteforce_odd_grid():
    """Brute force vs factorised on a ragged grid and a small head dim."""
    rng = np.random.default_rng(11)
    T, H, W, d = 3, 2, 5, 12
    N = T * H * W
    q, k, v, g = (rng.standard_normal((2, N, 1, d)) for _ in range(4))
    beta = rng.uniform(0.05, 0.95, (2, N, 1))
    args = (q, k, v, beta, g, T, H, W, 50.0, 1e-4, 2)
    f = O.forward(*args)
    bf = O.forward_bruteforce(*args)
    _close(f["pre"], bf["pre"], 1e-12, "odd-grid brute force")


def check_denominator_positive():
    """[V1]: without RoPE in the denominator every pair term k_pls_n . q_pls_j
    is >= 0, so den >= eps for every token.  Negative control: the same terms
    taken over rotated features are negative for some pairs, so a rotated
    denominator would carry no such guarantee."""
    rng = np.random.default_rng(3)
    T, H, W, d = 4, 6, 6, 32
    N = T * H * W
    q, k, v, g = (rng.standard_normal((1, N, 2, d)) for _ in range(4))
    beta = rng.uniform(0.0, 1.0, (1, N, 2))
    eps = 1e-6
    r = O.forward(q, k, v, beta, g, T, H, W, 10000.0, eps)
    assert np.all(r["den"] >= eps), "denominator below eps"
    ang = O.rope_angles(d, T, H, W, 10000.0)
    q_pls, q_til = O.feature_maps(q, ang)
    k_pls, k_til = O.feature_maps(k, ang)
    assert np.all(np.einsum("bnhc,bjhc->bnjh", k_pls, q_pls) >= 0.0)
    assert np.any(np.einsum("bnhc,bjhc->bnjh", k_til, q_til) < 0.0), \
        "negative control: every rotated pair term stayed non-negative"


def check_time_shift_invariance():
    """Dot products of rotated features depend on position differences only,
    and the denominator has no rotation, so a global time offset leaves the
    bidirectional output unchanged."""
    wl = workloads.WORKLOADS["tiny"]
    x = _inputs_f64(wl)
    args = (x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W, wl.rope_theta, wl.eps)
    a = O.forward(*args, t0=0)
    b = O.forward(*args, t0=7)
    _close(b["out"], a["out"], 1e-11, "time-shift invariance")


def check_rotation_preserves_norm():
    wl = workloads.WORKLOADS["tiny"]
    x = _inputs_f64(wl)
    ang = O.rope_angles(wl.head_dim, wl.T, wl.H, wl.W, wl.rope_theta)
    q_pls, q_til = O.feature_maps(x["q"], ang)
    assert np.allclose(np.linalg.norm(q_pls, axis=-1), np.linalg.norm(q_til, axis=-1),
                       rtol=1e-13, atol=0)


def check_plain_relu_linear_attention():
    """RoPE off, beta = 1 and g = +30 (sigma = 1 - 9.4e-14): the operator is
    plain ReLU linear attention on the normalised q/k ([V1]: SANA's ReLU
    linear attention), written here in textbook matrix form
        phi(Q) (phi(K)^T V) / (phi(Q) (phi(K)^T 1) + eps),
    followed by the output RMSNorm."""
    wl = workloads.WORKLOADS["tiny"]
    x = _inputs_f64(wl)
    beta = np.ones_like(x["beta"])
    g = np.full_like(x["g"], 30.0)
    r = O.forward(x["q"], x["k"], x["v"], beta, g, wl.T, wl.H, wl.W, 0.0, wl.eps)
    for h in range(wl.heads):
        Q, K, V = (x[n][0, :, h, :] for n in ("q", "k", "v"))
        nq = np.maximum(Q / np.sqrt((Q ** 2).mean(1, keepdims=True) + EPS_N), 0)
        nk = np.maximum(K / np.sqrt((K ** 2).mean(1, keepdims=True) + EPS_N), 0)
        num = nq @ (nk.T @ V)
        den = nq @ (nk.T @ np.ones((nk.shape[0], 1))) + wl.eps
        la = num / den
        want = la / np.sqrt((la ** 2).mean(1, keepdims=True) + EPS_N)
        _close(r["out"][0, :, h, :], want, 1e-11, "plain ReLU linear attention")


def check_gate_and_write_scale_invariance():
    """A uniform write gate c_b and a uniform output gate sigma scale every
    gated read-out x_j by the same constant c, and the output RMSNorm (gate
    before the norm) then gives out_b = out_a sqrt((ms + e_n) / (ms + e_n/c^2))
    with ms = mean(x_a^2) per token.  Every output row has RMS
    sqrt(ms / (ms + e_n))."""
    wl = workloads.WORKLOADS["tiny"]
    x = _inputs_f64(wl)
    base = (x["q"], x["k"], x["v"])
    geo = (wl.T, wl.H, wl.W, wl.rope_theta, wl.eps)
    a = O.forward(*base, np.full_like(x["beta"], 0.3), np.zeros_like(x["g"]), *geo)
    b = O.forward(*base, np.full_like(x["beta"], 0.9), np.full_like(x["g"], 30.0), *geo)
    c = (0.9 / 0.3) * (1.0 / (1.0 + math.exp(-30.0))) / 0.5
    _close(b["x"], c * a["x"], 1e-12, "uniform gates scale x")
    ms = np.mean(a["x"] ** 2, axis=-1, keepdims=True)
    _close(b["out"], a["out"] * np.sqrt((ms + EPS_N) / (ms + EPS_N / c ** 2)), 1e-12,
           "output norm after uniform gates")
    rms_out = np.sqrt(np.mean(a["out"] ** 2, axis=-1, keepdims=True))
    _close(rms_out, np.sqrt(ms / (ms + EPS_N)), 1e-12, "output row RMS")


# ---------------------------------------------------------------- block-causal

def _blk_inputs():
    rng = np.random.default_rng(21)
    nb, T_blk, H, W, d = 4, 2, 3, 4, 8
    N = nb * T_blk * H * W
    q, k, v, g = (rng.standard_normal((1, N, 2, d)) for _ in range(4))
    beta = rng.uniform(0.0, 1.0, (1, N, 2))
    return (q, k, v, beta, g), (nb, T_blk, H, W)


def check_block_causal_bruteforce():
    """[BLK]: the carried (S, z) form equals the prefix-masked pair sum where
    token j sees token n iff block(n) <= block(j)."""
    (q, k, v, beta, g), (nb, T_blk, H, W) = _blk_inputs()
    c = O.block_causal_forward(q, k, v, beta, g, nb, T_blk, H, W, 10000.0, 1e-5)
    bf = O.block_causal_bruteforce(q, k, v, beta, g, nb, T_blk, H, W, 10000.0, 1e-5)
    _close(c["out"], bf["out"], 1e-11, "block-causal vs prefix-masked brute force")


def check_block_causal_final_state():
    """After the last block the carried state is the full-sequence state and
    the last block's output is the bidirectional output of those tokens."""
    (q, k, v, beta, g), (nb, T_blk, H, W) = _blk_inputs()
    c = O.block_causal_forward(q, k, v, beta, g, nb, T_blk, H, W, 10000.0, 1e-5)
    f = O.forward(q, k, v, beta, g, nb * T_blk, H, W, 10000.0, 1e-5)
    _close(c["S"], f["S"], 1e-12, "final block state")
    _close(c["z"], f["z"], 1e-12, "final key sum")
    L = T_blk * H * W
    _close(c["out"][:, -L:], f["out"][:, -L:], 1e-11, "last block = bidirectional")


def _causal_inputs(H=3, W=2, T=4, d=8, seed=31):
    rng = np.random.default_rng(seed)
    N = T * H * W
    q, k, v, g = (rng.standard_normal((2, N, 2, d)) for _ in range(4))
    beta = rng.uniform(0.0, 1.0, (2, N, 2))
    return (q, k, v, beta, g), (T, H, W)


def check_causal_bruteforce():
    """Token-level causal ([BLK] running sums): equals the pair sum where
    token j sees token n iff n <= j."""
    (q, k, v, beta, g), (T, H, W) = _causal_inputs()
    c = O.causal_forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    bf = O.causal_bruteforce(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    _close(c["out"], bf["out"], 1e-11, "causal vs prefix-masked brute force")
    _close(c["x"], bf["x"], 1e-11, "causal gated read-out vs brute force")


def check_causal_last_token_sees_everything():
    """The last token's prefix is the whole sequence: its output is the
    bidirectional output."""
    (q, k, v, beta, g), (T, H, W) = _causal_inputs()
    c = O.causal_forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    f = O.forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    _close(c["out"][:, -1], f["out"][:, -1], 1e-11, "causal last token = bidirectional")


def check_causal_first_token_alone():
    """The first token sees only itself: its output is the one-token
    operator on that token, whatever follows."""
    (q, k, v, beta, g), (T, H, W) = _causal_inputs()
    c = O.causal_forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    one = O.forward(q[:, :1], k[:, :1], v[:, :1], beta[:, :1], g[:, :1], 1, 1, 1, 10000.0, 1e-5)
    _close(c["out"][:, 0], one["out"][:, 0], 1e-12, "causal first token = single token")


def check_causal_is_one_token_blocks():
    """With one token per frame (H = W = 1), token-level causal equals the
    block-causal carry with one-frame blocks."""
    (q, k, v, beta, g), (T, H, W) = _causal_inputs(H=1, W=1, T=9)
    c = O.causal_forward(q, k, v, beta, g, T, 1, 1, 10000.0, 1e-5)
    b = O.block_causal_forward(q, k, v, beta, g, T, 1, 1, 1, 10000.0, 1e-5)
    _close(c["out"], b["out"], 1e-11, "causal = one-token blocks")


def check_causal_time_shift_invariance():
    """ReLU before RoPE: numerators depend on position differences only, so a
    global time shift leaves the causal output unchanged ([V1])."""
    (q, k, v, beta, g), (T, H, W) = _causal_inputs()
    a = O.causal_forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5, t0=0)
    b = O.causal_forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5, t0=7)
    _close(a["out"], b["out"], 1e-10, "causal time shift")


def check_causal_at_selected_tokens():
    """The token-by-token prefix form at selected tokens equals the running
    sums (two computations of the same definition: per-token prefixes
    against cumulative sums), and its end state is the full-sequence state."""
    (q, k, v, beta, g), (T, H, W) = _causal_inputs()
    toks = [0, 1, 5, 11, T * H * W - 1]
    a = O.causal_forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    b = O.causal_forward_at(q, k, v, beta, g, T, H, W, 10000.0, 1e-5, toks)
    for key in ("den", "pre", "out"):
        _close(b[key], a[key][:, toks], 1e-12, f"causal at tokens: {key}")
    full = O.forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    _close(b["S_end"], full["S"], 1e-12, "causal end state")
    _close(b["z_end"], full["z"], 1e-12, "causal end key sum")


def check_causal_carried_state():
    """Streaming: running the second half of a sequence from the first
    half's end state (with the time offset of the second half) gives the
    whole sequence's causal outputs for the second half."""
    (q, k, v, beta, g), (T, H, W) = _causal_inputs(T=4)
    L = (T // 2) * H * W
    whole = O.causal_forward(q, k, v, beta, g, T, H, W, 10000.0, 1e-5)
    first = O.causal_forward_at(q[:, :L], k[:, :L], v[:, :L], beta[:, :L], g[:, :L], T // 2,
                                H, W, 10000.0, 1e-5, [L - 1])
    sl = slice(L, None)
    second = O.causal_forward_at(q[:, sl], k[:, sl], v[:, sl], beta[:, sl], g[:, sl], T // 2,
                                 H, W, 10000.0, 1e-5, range(L), t0=T // 2,
                                 S0=first["S_end"], z0=first["z_end"])
    _close(second["out"], whole["out"][:, L:], 1e-12, "carried causal state")


# ---------------------------------------------------- gated softmax anchor

def check_anchor_one_token():
    """N = 1: the softmax of one score is 1, so out = sigmoid(g) * v exactly."""
    rng = np.random.default_rng(8)
    q, k, v, g = (rng.standard_normal((1, 1, 2, 8)) for _ in range(4))
    r = O.softmax_anchor(q, k, v, g, 1, 1, 1, 1e4)
    _close(r["out"], (1 / (1 + np.exp(-g))) * v, 1e-15, "anchor, one token")


def check_anchor_two_token_closed_form():
    """T = 2, H = W = 1, d = 2, RoPE off: q0 = (1, 0) -> q_hat0 = (1, 0) /
    sqrt(0.5 + e_n) ~ (sqrt2, 0); k0 = (1, 0), k1 = (0, 1) likewise; scores of
    token 0: (c^2 / sqrt2, 0) with c = 1/sqrt(0.5 + e_n); weights
    (e^a, 1) / (e^a + 1); out = sigma(g) * weighted v."""
    e_n = 1e-6
    c = 1 / math.sqrt(0.5 + e_n)
    q = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    k = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, -1.0]]).reshape(1, 2, 1, 2)
    g = np.zeros((1, 2, 1, 2))
    a = c * c / math.sqrt(2)
    w0 = np.array([math.exp(a), 1.0]) / (math.exp(a) + 1.0)
    want0 = 0.5 * (w0[0] * np.array([1.0, 2.0]) + w0[1] * np.array([3.0, -1.0]))
    r = O.softmax_anchor(q, k, v, g, 2, 1, 1, 0.0)
    _close(r["out"][0, 0, 0], want0, 1e-14, "anchor token 0")
    want1 = 0.5 * (w0[1] * np.array([1.0, 2.0]) + w0[0] * np.array([3.0, -1.0]))
    _close(r["out"][0, 1, 0], want1, 1e-14, "anchor token 1")


def check_anchor_matches_library_sdpa():
    """On the normalised, rotated q and k (the oracle's own feature maps are
    pinned above), the attention equals torch's scaled_dot_product_attention
    in fp64."""
    import torch
    rng = np.random.default_rng(9)
    T, H, W, d, Hh = 2, 3, 2, 16, 2
    N = T * H * W
    q, k, v, g = (rng.standard_normal((1, N, Hh, d)) for _ in range(4))
    r = O.softmax_anchor(q, k, v, g, T, H, W, 1e4)
    ang = O.rope_angles(d, T, H, W, 1e4)
    qt = O.rope_rotate(O.rms_normalize(q), ang)
    kt = O.rope_rotate(O.rms_normalize(k), ang)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a.transpose(0, 2, 1, 3)))
    lib = torch.nn.functional.scaled_dot_product_attention(to(qt), to(kt), to(v))
    _close(r["attn"], lib.numpy().transpose(0, 2, 1, 3), 1e-12, "anchor vs torch SDPA")


def check_anchor_time_shift_invariance():
    """RoPE makes q_til . k_til depend on position differences only, so a
    global time offset t0 leaves the anchor's output unchanged (both q and k
    rotated the same way, by the same positions)."""
    rng = np.random.default_rng(12)
    T, H, W, d, Hh = 3, 2, 2, 16, 2
    N = T * H * W
    q, k, v, g = (rng.standard_normal((1, N, Hh, d)) for _ in range(4))
    a = O.softmax_anchor(q, k, v, g, T, H, W, 1e4, t0=0)["out"]
    b = O.softmax_anchor(q, k, v, g, T, H, W, 1e4, t0=7)["out"]
    _close(b, a, 1e-11, "anchor under a time shift")
    c = O.softmax_anchor(q, k, v, g, T, H, W, 0.0, t0=0)["out"]
    assert np.max(np.abs(c - a)) > 1e-3, "RoPE must change the anchor's output"


def check_anchor_uniform_scores():
    """q = 0 gives q_hat = 0 and all scores 0: every token reads the mean of v."""
    rng = np.random.default_rng(10)
    k, v, g = (rng.standard_normal((1, 6, 1, 4)) for _ in range(3))
    q = np.zeros((1, 6, 1, 4))
    r = O.softmax_anchor(q, k, v, g, 1, 2, 3, 1e4)
    _close(r["attn"][0, :, 0], np.repeat(v[0, :, 0].mean(axis=0, keepdims=True), 6, axis=0),
           1e-14, "uniform attention")


def check_anchor_query_rows():
    """Selected query rows (queries=...) equal a per-row brute force: for each
    chosen token j, scores over all n by explicit dot products, max-shifted
    exponentials, normalised weights, weighted sum of v, times sigmoid(g_j)."""
    rng = np.random.default_rng(11)
    T, H, W, d, Hh = 2, 2, 3, 8, 2
    N = T * H * W
    q, k, v, g = (rng.standard_normal((1, N, Hh, d)) for _ in range(4))
    rows = [0, 5, 11, 7]
    r = O.softmax_anchor(q, k, v, g, T, H, W, 1e4, queries=rows)
    ang = O.rope_angles(d, T, H, W, 1e4)
    qt = O.rope_rotate(O.rms_normalize(q), ang)
    kt = O.rope_rotate(O.rms_normalize(k), ang)
    for i, j in enumerate(rows):
        for h in range(Hh):
            sc = [sum(qt[0, j, h, c] * kt[0, n, h, c] for c in range(d)) / math.sqrt(d)
                  for n in range(N)]
            m = max(sc)
            w = [math.exp(x - m) for x in sc]
            tot = sum(w)
            attn = [sum(w[n] * v[0, n, h, c] for n in range(N)) / tot for c in range(d)]
            gate = 1 / (1 + np.exp(-g[0, j, h]))
            _close(r["out"][0, i, h], gate * np.array(attn), 1e-13, f"anchor row {j} head {h}")


# ------------------------------------------------ the layer's projections

def check_project_in_layout():
    """One token, C = 2, Hh = 2, d = 2: W_in rows in the order q (4 rows), k,
    v, g, then 2 beta-logit rows.  With x = (1, 2) each output is its row's
    dot with x; q of head 1 is rows 2..3; beta = sigmoid of the last two."""
    Hh, d, C = 2, 2, 2
    rows = 4 * Hh * d + Hh
    W_in = np.zeros((rows, C))
    for r in range(rows):
        W_in[r] = (r, 1.0)                 # row r . (1, 2) = r + 2
    x = np.array([[[1.0, 2.0]]])
    p = O.project_in(x, W_in, Hh, d)
    want = {"q": [2, 3, 4, 5], "k": [6, 7, 8, 9], "v": [10, 11, 12, 13], "g": [14, 15, 16, 17]}
    for name, w in want.items():
        _close(p[name].ravel(), w, 0.0, f"project_in {name}")
    assert p["q"].shape == (1, 1, Hh, d)
    _close(p["q"][0, 0, 1], [4, 5], 0.0, "q of head 1")
    _close(p["beta"].ravel(), [1 / (1 + math.exp(-18)), 1 / (1 + math.exp(-19))], 1e-15,
           "beta = sigmoid(logits)")


def check_project_out_layout():
    """o [1, 1, Hh=2, d=2] = (1, 2 | 3, 4) flattened head-major; W_o rows pick
    single entries: W_o = [[0,0,1,0], [1,1,1,1]] -> (3, 10)."""
    o = np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 1, 2, 2)
    W_o = np.array([[0.0, 0.0, 1.0, 0.0], [1.0, 1.0, 1.0, 1.0]])
    _close(O.project_out(o, W_o).ravel(), [3.0, 10.0], 0.0, "project_out")


def check_layer_is_the_composition():
    """layer_forward = W_o applied to the operator of the projections."""
    rng = np.random.default_rng(3)
    Hh, d, C, T, H, W = 2, 8, 6, 2, 2, 2
    N = T * H * W
    x = rng.standard_normal((1, N, C))
    W_in = rng.standard_normal((4 * Hh * d + Hh, C)) * 0.3
    W_o = rng.standard_normal((5, Hh * d))
    r = O.layer_forward(x, W_in, W_o, Hh, d, T, H, W, 1e4, 1e-5)
    y = x @ W_in.T
    q, k, v, g = (y[..., i * Hh * d:(i + 1) * Hh * d].reshape(1, N, Hh, d) for i in range(4))
    beta = 1 / (1 + np.exp(-y[..., 4 * Hh * d:]))
    op = O.forward(q, k, v, beta, g, T, H, W, 1e4, 1e-5)
    _close(r["y"], op["out"].reshape(1, N, Hh * d) @ W_o.T, 1e-12, "layer composition")


# ---------------------------------------------------- MXFP8 input decoding

def check_e4m3_format_values():
    """Values the OCP FP8 E4M3 definition fixes: 1.0, -2.0, the largest
    finite 448, the smallest normal 2^-6, the largest subnormal 7/8 * 2^-6,
    the smallest subnormal 2^-9, signed zeros and the NaN codes."""
    want = {0x38: 1.0, 0xC0: -2.0, 0x7E: 448.0, 0xFE: -448.0, 0x08: 2.0 ** -6,
            0x07: 0.875 * 2.0 ** -6, 0x01: 2.0 ** -9, 0x00: 0.0, 0x3C: 1.5, 0x44: 3.0}
    got = O.e4m3_decode(np.array(list(want), dtype=np.uint8))
    _close(got, list(want.values()), 0.0, "e4m3 values")
    assert np.signbit(O.e4m3_decode(np.array([0x80], dtype=np.uint8)))[0], "0x80 is -0"
    assert np.isnan(O.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all(), "NaN codes"


def check_e4m3_matches_library():
    """All 256 codes against torch's float8_e4m3fn conversion."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(lib)), "e4m3 NaN codes differ"
    ok = ~np.isnan(lib)
    assert np.array_equal(got[ok], lib[ok]), "e4m3 decode differs from torch"


def check_e8m0_matches_library():
    """All 256 scale codes against torch's float8_e8m0fnu conversion."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = O.e8m0_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(lib)), "e8m0 NaN codes differ"
    ok = ~np.isnan(lib)
    assert np.array_equal(got[ok], lib[ok]), "e8m0 decode differs from torch"


def check_mx_block_layout():
    """A 64-element row with scales 2^1 and 2^-3: elements 0..31 take the
    first, 32..63 the second."""
    codes = np.full((1, 64), 0x38, dtype=np.uint8)          # every element 1.0
    scales = np.array([[128, 124]], dtype=np.uint8)         # 2^1, 2^-3
    got = O.mx_dequantize(codes, scales)
    _close(got[0, :32], [2.0] * 32, 0.0, "first block")
    _close(got[0, 32:], [0.125] * 32, 0.0, "second block")


def check_mx_forward_row_scale_invariance():
    """Scaling every block scale of a q (or k) row by the same power of two
    leaves the output unchanged up to the RMSNorm epsilon: the operator sees
    q and k only through their RMS-normalised values."""
    rng = np.random.default_rng(57)
    T, H, W, d = 2, 2, 3, 64
    N = T * H * W
    codes = {n: rng.integers(0, 0x77, (1, N, 2, d)).astype(np.uint8) |
             (rng.integers(0, 2, (1, N, 2, d)).astype(np.uint8) << 7) for n in "qkvg"}
    scales = {n: rng.integers(120, 130, (1, N, 2, d // O.MX_BLOCK)).astype(np.uint8) for n in "qkv"}
    scales["g"] = rng.integers(118, 122, (1, N, 2, d // O.MX_BLOCK)).astype(np.uint8)   # |g| < 15
    beta = rng.uniform(0.0, 1.0, (1, N, 2))
    args = lambda sc: [(codes[n], sc[n]) for n in "qkv"]
    a = O.forward_mx(*args(scales), beta, (codes["g"], scales["g"]), T, H, W, 1e4, 1e-5)
    shifted = dict(scales, q=scales["q"] + 3, k=scales["k"] - 2)
    b = O.forward_mx(*args(shifted), beta, (codes["g"], scales["g"]), T, H, W, 1e4, 1e-5)
    _close(b["out"], a["out"], 1e-5, "row scale invariance")


# ------------------------------------------------------ tolerance metrics
#
# Every GPU pass/fail goes through these four functions, so each is pinned to
# values worked out by hand (and the bf16 spacing to torch's bf16 rounding):
# a slip in one of them (the RMS of the wrong array, a lost abs, a wrong
# exponent) would otherwise loosen every parity test without anything failing.

_REF4 = np.array([3.0, -4.0, 0.0, 0.0])        # rms = sqrt((9 + 16) / 4) = 2.5


def check_metric_max_err_over_rms():
    """max|got - ref| / rms(ref): errors (0.1, 0, 0, -0.3) give 0.3 / 2.5."""
    got = _REF4 + np.array([0.1, 0.0, 0.0, -0.3])
    _close(O.max_err_over_rms(got, _REF4), 0.12, 1e-12, "max_err_over_rms")
    _close(O.max_err_over_rms(_REF4 + np.array([0.0, 0.5, 0.0, 0.0]), _REF4), 0.2, 1e-12,
           "max_err_over_rms, one error")
    assert O.max_err_over_rms(_REF4, _REF4) == 0.0


def check_metric_rel_rms_floor():
    """max |got - ref| / max(|ref|, rms(ref)) with rms(ref) = 2.5:
    errors (0.6, -1.0, 0.3, -0.8) give 0.6/3, 1.0/4, 0.3/2.5, 0.8/2.5, max 0.32;
    a single error -2 on the 4 gives 2/4 (relative above the RMS)."""
    got = _REF4 + np.array([0.6, -1.0, 0.3, -0.8])
    _close(O.max_rel_err_rms_floor(got, _REF4), 0.32, 1e-12, "rel err with RMS floor")
    got = _REF4 + np.array([0.0, -2.0, 0.0, 0.0])
    _close(O.max_rel_err_rms_floor(got, _REF4), 0.5, 1e-12, "rel err above the RMS")


def check_metric_row_rms():
    """Per-row errors over per-row RMS: rows (3, -4, 0, 0) (rms 2.5) and
    (30, -40, 0, 0) (rms 25) with errors (0, 0.5, 0, 0) and (1, 0, 0, -2)
    give max(0.5/2.5, 2/25) = 0.2; a global RMS would give 2/17.77."""
    ref = np.array([[3.0, -4.0, 0.0, 0.0], [30.0, -40.0, 0.0, 0.0]])
    got = ref + np.array([[0.0, 0.5, 0.0, 0.0], [1.0, 0.0, 0.0, -2.0]])
    _close(O.max_err_over_row_rms(got, ref), 0.2, 1e-12, "row-RMS metric")
    got = ref + np.array([[0.0, 0.0, 0.0, 0.0], [0.0, 0.0, 0.0, -5.0]])
    _close(O.max_err_over_row_rms(got, ref), 0.2, 1e-12, "row-RMS metric, second row")


def check_metric_bf16_half_ulp():
    """Half the bf16 spacing (8 significant bits) at hand-picked values, then
    against torch's round-to-nearest-even bf16 conversion: a value halfway
    between two bf16 neighbours is exactly half a spacing from its rounding."""
    import torch
    vals = np.array([1.0, 1.99, 4.0, 7.99, 0.75, -3.0, 2.0 ** 20])
    want = np.array([2.0 ** -8, 2.0 ** -8, 2.0 ** -6, 2.0 ** -6, 2.0 ** -9, 2.0 ** -7, 2.0 ** 12])
    _close(O.bf16_half_ulp(vals), want, 0.0, "bf16 half ulp")
    rng = np.random.default_rng(5)
    e = rng.integers(-60, 60, 400)
    m = rng.integers(0, 128, 400)
    x = np.ldexp(1.0 + (2 * m + 1) / 256.0, e) * np.where(rng.random(400) < 0.5, -1.0, 1.0)
    rounded = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    _close(np.abs(rounded - x), O.bf16_half_ulp(x), 0.0, "midpoints vs torch bf16")


def check_metric_rel_rms_bf16out():
    """Error beyond half a bf16 spacing, over rms(ref) = 2.5.  Half spacings:
    2^-7 at 3, 2^-6 at 4.  Errors (2^-7, -0.025, 0, 0) exceed them by
    (0, 0.025 - 2^-6, 0, 0): 0.009375 / 2.5 = 0.00375."""
    got = _REF4 + np.array([2.0 ** -7, -0.025, 0.0, 0.0])
    _close(O.bf16_out_err_over_rms(got, _REF4), 0.00375, 1e-9, "bf16 output metric")
    got = _REF4 + np.array([2.0 ** -7, -2.0 ** -6, 0.0, 0.0])
    assert O.bf16_out_err_over_rms(got, _REF4) == 0.0, "a correct rounding scores 0"


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
