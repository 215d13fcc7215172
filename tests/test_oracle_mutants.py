"""Plant plausible mistakes in the oracle (on the CPU) and verify that the
pins catch every one of them: each mutant must fail at least one check."""
import numpy as np
import pytest

import oracle.gla_oracle as O
import oracle_pins

_orig = {name: getattr(O, name) for name in dir(O) if not name.startswith("_")}


def _rotate_backwards(x, angles):
    return _orig["rope_rotate"](x, -angles)


def _rope_before_relu(x, angles):
    x_hat = O.rms_normalize(x)
    if angles is None:
        p = O.relu(x_hat)
        return p, p
    return O.relu(x_hat), O.relu(_orig["rope_rotate"](x_hat, angles))


def _beta_in_keysum(k_til, k_pls, v, beta):
    S, _ = _orig["state_and_keysum"](k_til, k_pls, v, beta)
    return S, (beta[..., None] * k_pls).sum(axis=1)


def _transposed_state(k_til, k_pls, v, beta):
    S, z = _orig["state_and_keysum"](k_til, k_pls, v, beta)
    return np.swapaxes(S, -1, -2), z


def _rotated_keysum(k_til, k_pls, v, beta):
    return _orig["state_and_keysum"](k_til, k_til, v, beta)


def _gate_after_norm(S, z, q_pls, q_til, g, eps):
    r = _orig["read_out"](S, z, q_pls, q_til, g, eps)
    r["out"] = O.sigmoid(g) * O.rms_normalize(r["pre"])
    return r


def _no_eps_in_den(S, z, q_pls, q_til, g, eps):
    return _orig["read_out"](S, z, q_pls, q_til, g, 0.0)


def _unnormalised_keysum(k_til, k_pls, v, beta):
    return _orig["state_and_keysum"](k_til, np.abs(k_pls) * 1.5, v, beta)


def _rms_sum(x):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + O.RMS_EPS)


def _rms_no_eps(x):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True))


def _freq_doubled(d, T, H, W, rope_theta, t0=0):
    return _orig["rope_angles"](d, T, H, W, rope_theta ** 2, t0)


def _axes_swapped(T, H, W, t0=0):
    t, h, w = _orig["token_positions"](T, H, W, t0)
    return t, w, h


def _no_time_offset(T, H, W, t0=0):
    return _orig["token_positions"](T, H, W, 0)


def _exclusive_block(S, z, q, k, v, beta, g, T_blk, H, W, t0, rope_theta, eps):
    d = q.shape[-1]
    angles = None if rope_theta <= 0 else O.rope_angles(d, T_blk, H, W, rope_theta, t0)
    q_pls, q_til = O.feature_maps(q, angles)
    k_pls, k_til = O.feature_maps(k, angles)
    dS, dz = O.state_and_keysum(k_til, k_pls, v, beta)
    r = O.read_out(S + 0.0, z + eps, q_pls, q_til, g, eps)   # reads the old state
    r.update(S=S + dS, z=z + dz)
    return r


def _neg_sigmoid(x):
    return 1.0 / (1.0 + np.exp(x))


def _causal_exclusive(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=0):
    """Token j reads the running sums over tokens 0..j-1 only (the printed
    sum_{j<i} taken literally)."""
    d = q.shape[-1]
    angles = None if rope_theta <= 0 else O.rope_angles(d, T, H, W, rope_theta, t0)
    q_pls, q_til = O.feature_maps(q, angles)
    k_pls, k_til = O.feature_maps(k, angles)
    B, N, Hh, _ = q.shape
    pre = np.empty_like(q)
    dens = np.empty((B, N, Hh))
    for b in range(B):
        for h in range(Hh):
            per = v[b, :, h, :, None] * (beta[b, :, h, None, None] * k_til[b, :, h, None, :])
            S_run = np.cumsum(per, axis=0) - per
            z_run = np.cumsum(k_pls[b, :, h, :], axis=0) - k_pls[b, :, h, :]
            den = np.einsum("nc,nc->n", z_run, q_pls[b, :, h, :]) + eps
            dens[b, :, h] = den
            pre[b, :, h, :] = np.einsum("nac,nc->na", S_run, q_til[b, :, h, :]) / den[:, None]
    x = O.sigmoid(g) * pre
    return dict(den=dens, pre=pre, x=x, out=O.rms_normalize(x))


def _causal_suffix(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=0):
    """Running sums taken from the end of the sequence instead of the start."""
    flip = lambda a: a[:, ::-1]
    r = _orig["causal_forward"](flip(q), flip(k), flip(v), flip(beta), flip(g), T, H, W,
                                rope_theta, eps, t0)
    return {key: flip(val) for key, val in r.items()}


def _causal_at_exclusive(q, k, v, beta, g, T, H, W, rope_theta, eps, tokens, t0=0, S0=None,
                         z0=None):
    """Each selected token read out against the tokens before it only."""
    tokens = list(tokens)
    r = _orig["causal_forward_at"](q, k, v, beta, g, T, H, W, rope_theta, eps,
                                   [max(j - 1, 0) for j in tokens], t0, S0, z0)
    return r


def _causal_at_no_carry(q, k, v, beta, g, T, H, W, rope_theta, eps, tokens, t0=0, S0=None,
                        z0=None):
    """The carried-in state dropped."""
    return _orig["causal_forward_at"](q, k, v, beta, g, T, H, W, rope_theta, eps, tokens, t0)


def _project_in_no_sigmoid(x, W_in, heads, head_dim):
    p = _orig["project_in"](x, W_in, heads, head_dim)
    y = x @ W_in.T
    p["beta"] = y[..., 4 * heads * head_dim:4 * heads * head_dim + heads]
    return p


def _project_in_qk_swapped(x, W_in, heads, head_dim):
    p = _orig["project_in"](x, W_in, heads, head_dim)
    p["q"], p["k"] = p["k"], p["q"]
    return p


def _project_out_transposed(o, W_o):
    B, N, Hh, d = o.shape
    return np.swapaxes(o, 2, 3).reshape(B, N, Hh * d) @ W_o.T


def _anchor_gate_inside(q, k, v, g, T, H, W, rope_theta, t0=0, queries=None):
    r = _orig["softmax_anchor"](q, k, v * (1 / (1 + np.exp(-g))), np.full_like(g, 40.0), T, H, W,
                                rope_theta, t0, queries)
    return r


def _anchor_k_rotated_backwards(q, k, v, g, T, H, W, rope_theta, t0=0, queries=None):
    ang = O.rope_angles(q.shape[-1], T, H, W, rope_theta, t0) if rope_theta > 0 else None
    if ang is None:
        return _orig["softmax_anchor"](q, k, v, g, T, H, W, rope_theta, t0, queries)
    qt = O.rope_rotate(O.rms_normalize(q), ang)
    kt = O.rope_rotate(O.rms_normalize(k), -ang)
    return _orig["softmax_anchor"](qt, kt, v, g, T, H, W, 0.0, t0, queries)


def _anchor_softmax_over_queries(q, k, v, g, T, H, W, rope_theta, t0=0, queries=None):
    return _orig["softmax_anchor"](k, q, v, g, T, H, W, rope_theta, t0, queries)


def _e4m3_bias8(codes):
    return _orig["e4m3_decode"](codes) / 2.0


def _e4m3_no_subnormals(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    out = _orig["e4m3_decode"](codes)
    sub = ((c >> 3) & 0xF) == 0
    m = (c & 0x7).astype(np.float64)
    out[sub] = np.where(c[sub] & 0x80, -1.0, 1.0) * (1.0 + m[sub] / 8.0) * 2.0 ** -7
    return out


def _e8m0_bias128(codes):
    return _orig["e8m0_decode"](codes) / 2.0


def _mx_scales_tiled(codes, scales):
    x = O.e4m3_decode(codes)
    sc = O.e8m0_decode(scales)
    return x * np.tile(sc, (1,) * (sc.ndim - 1) + (O.MX_BLOCK,))


MUTANTS = {
    "rope_backwards": ("rope_rotate", _rotate_backwards),
    "rope_before_relu": ("feature_maps", _rope_before_relu),
    "beta_in_keysum": ("state_and_keysum", _beta_in_keysum),
    "state_transposed": ("state_and_keysum", _transposed_state),
    "rotated_keysum": ("state_and_keysum", _rotated_keysum),
    "gate_after_norm": ("read_out", _gate_after_norm),
    "no_eps_in_den": ("read_out", _no_eps_in_den),
    "keysum_wrong_features": ("state_and_keysum", _unnormalised_keysum),
    "rmsnorm_sum": ("rms_normalize", _rms_sum),
    "rmsnorm_no_eps": ("rms_normalize", _rms_no_eps),
    "rope_freq_wrong": ("rope_angles", _freq_doubled),
    "rope_axes_swapped": ("token_positions", _axes_swapped),
    "rope_no_time_offset": ("token_positions", _no_time_offset),
    "block_exclusive": ("block_causal_step", _exclusive_block),
    "sigmoid_sign": ("sigmoid", _neg_sigmoid),
    "causal_exclusive": ("causal_forward", _causal_exclusive),
    "causal_suffix": ("causal_forward", _causal_suffix),
    "causal_at_exclusive": ("causal_forward_at", _causal_at_exclusive),
    "causal_at_no_carry": ("causal_forward_at", _causal_at_no_carry),
    "project_in_no_sigmoid": ("project_in", _project_in_no_sigmoid),
    "project_in_qk_swapped": ("project_in", _project_in_qk_swapped),
    "project_out_channel_major": ("project_out", _project_out_transposed),
    "anchor_gate_on_values": ("softmax_anchor", _anchor_gate_inside),
    "anchor_q_k_swapped": ("softmax_anchor", _anchor_softmax_over_queries),
    "anchor_k_rotated_backwards": ("softmax_anchor", _anchor_k_rotated_backwards),
    "e4m3_bias8": ("e4m3_decode", _e4m3_bias8),
    "e4m3_no_subnormals": ("e4m3_decode", _e4m3_no_subnormals),
    "e8m0_bias128": ("e8m0_decode", _e8m0_bias128),
    "mx_scales_tiled": ("mx_dequantize", _mx_scales_tiled),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check()
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"


# Mistakes in the tolerance metrics every GPU parity test goes through.

def _rms_of_got(got, ref):
    return _orig["max_err_over_rms"](ref, got)


def _err_no_abs(got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    return float(np.max(got - ref) / np.sqrt(np.mean(ref * ref)))


def _err_mean_abs(got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / np.mean(np.abs(ref)))


def _floor_no_abs(got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max((got - ref) / np.maximum(np.abs(ref), rms)))


def _floor_rms_of_got(got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    rms = np.sqrt(np.mean(got * got))
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), rms)))


def _floor_rms_only(got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref * ref)))


def _half_ulp_exp7(ref):
    a = np.maximum(np.abs(np.asarray(ref, dtype=np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, (np.floor(np.log2(a)) - 7).astype(int))


def _half_ulp_ceil(ref):
    a = np.maximum(np.abs(np.asarray(ref, dtype=np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, (np.ceil(np.log2(a)) - 8).astype(int))


def _bf16out_no_rounding_allowance(got, ref):
    return _orig["max_err_over_rms"](got, ref)


def _bf16out_rms_of_got(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    excess = np.maximum(np.abs(got - ref) - _orig["bf16_half_ulp"](ref), 0.0)
    return float(np.max(excess) / np.sqrt(np.mean(got * got)))


def _bf16out_full_ulp(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    excess = np.maximum(np.abs(got - ref) - 2.0 * _orig["bf16_half_ulp"](ref), 0.0)
    return float(np.max(excess) / np.sqrt(np.mean(ref * ref)))


def _row_rms_global(got, ref):
    return _orig["max_err_over_rms"](got, ref)


def _row_rms_of_got(got, ref):
    return _orig["max_err_over_row_rms"](ref, got)


METRIC_MUTANTS = {
    "row_rms_global": (O, "max_err_over_row_rms", _row_rms_global),
    "row_rms_of_got": (O, "max_err_over_row_rms", _row_rms_of_got),
    "err_rms_of_got": (O, "max_err_over_rms", _rms_of_got),
    "err_no_abs": (O, "max_err_over_rms", _err_no_abs),
    "err_mean_abs": (O, "max_err_over_rms", _err_mean_abs),
    "floor_no_abs": (O, "max_rel_err_rms_floor", _floor_no_abs),
    "floor_rms_of_got": (O, "max_rel_err_rms_floor", _floor_rms_of_got),
    "floor_missing": (O, "max_rel_err_rms_floor", _floor_rms_only),
    "half_ulp_exp7": (O, "bf16_half_ulp", _half_ulp_exp7),
    "half_ulp_ceil": (O, "bf16_half_ulp", _half_ulp_ceil),
    "bf16out_no_allowance": (O, "bf16_out_err_over_rms", _bf16out_no_rounding_allowance),
    "bf16out_rms_of_got": (O, "bf16_out_err_over_rms", _bf16out_rms_of_got),
    "bf16out_full_ulp": (O, "bf16_out_err_over_rms", _bf16out_full_ulp),
}


@pytest.mark.parametrize("name", sorted(METRIC_MUTANTS))
def test_metric_mutant_is_caught(name, monkeypatch):
    mod, attr, fn = METRIC_MUTANTS[name]
    monkeypatch.setattr(mod, attr, fn)
    failed = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check()
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(check.__name__)
    assert failed, f"metric mutant {name} passed every pin"
