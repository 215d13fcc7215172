"""Plain fp64 CPU oracle for gated bidirectional ReLU linear attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library (no kernels, headers, tables or helpers); the only thing both
sides see is the seeded input generator, which holds none of the method's
arithmetic.

What it computes, and where that is stated
------------------------------------------
Sources (web pages; cited by title and section):

[GBLA]  "SANA-Video 2.0: Hybrid Linear Attention with Attention Residuals for
        Efficient Video Generation" - paper.rainbus.top summary, prerequisites,
        "Gated Bilinear Linear Attention": the read-out
        o_j = W_o RMSNorm[ sigma(g_j) * (sum_n phi(k_n)^T phi(q_j) + eps)^-1 S q_j ]
        with phi = ReLU, RoPE applied to the normalised q/k, write gate beta,
        sigmoid output gate g, bidirectional (non-causal) sum.
[LA]    same page, prerequisites, "Linear Attention": the state
        S = sum_n v_n (beta_n k_n)^T in R^{d x d}.
[V1]    "SANA-Video: Efficient Video Generation with Block Linear Diffusion
        Transformer" - papernotes.org notes, method, key design 1 "Linear Video
        DiT": RoPE is applied after the ReLU, RoPE(phi(Q)), and only in the
        numerator, so the denominator stays positive.
[BLK]   same notes, key design 2 "block linear attention + constant-memory KV
        cache": causal linear attention only needs the running sums of the
        per-token states and of the key features, so a block carries (S, z).

Per head, with head dim d:
    q_hat = RMSNorm(q)      k_hat = RMSNorm(k)            (over d, no weight)
    q_pls = ReLU(q_hat)     k_pls = ReLU(k_hat)
    q_til = RoPE3D(q_pls)   k_til = RoPE3D(k_pls)         (numerator only)
    S     = sum_n v_n (beta_n k_til_n)^T                  (d x d)
    z     = sum_n k_pls_n                                  (d)
    den_j = z . q_pls_j + eps
    pre_j = S q_til_j / den_j
    x_j   = sigmoid(g_j) * pre_j
    o_j   = RMSNorm(x_j)                                   (W_o is outside)

Readings taken where the pages are silent (all listed in the design notes):
  * z and the denominator use the normalised, ReLU'd, un-rotated vectors.
  * ReLU before RoPE ([V1]); beta scales only the write into S ([LA], [GBLA]).
  * RMSNorm is per head over d with no affine weight; its epsilon is the fixed
    constant RMS_EPS = 1e-6.
  * 3D RoPE split (the pages give none): P = d/2 rotation pairs; the time axis
    gets P - 2*floor(P/3) pairs, height and width floor(P/3) each, as
    contiguous channel chunks in the order t, h, w.  Inside a chunk of p
    pairs, pair i is channels (2i, 2i+1) with frequency theta^(-i/p) and angle
    pos_axis * frequency; (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).
    Integer positions from 0, token order n = (t*H + h)*W + w; the time
    position is offset by t0 in the block-causal variant.  rope_theta <= 0
    turns RoPE off.
  * Block-causal: a token of block b sees every token of blocks 0..b
    (inclusive of its own block).  Token-level causal: token j sees tokens
    0..j (inclusive of itself).

Tensors are numpy float64 arrays: q, k, v, g are [B, N, Hh, d] and beta is
[B, N, Hh]; N = T*H*W.
"""
import numpy as np

RMS_EPS = 1e-6


# ---------------------------------------------------------------- elementwise

def rms_normalize(x):
    """RMSNorm over the last axis, no affine weight ([GBLA] normalised q/k and
    the output RMSNorm)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + RMS_EPS)


def relu(x):
    """phi = ReLU ([GBLA], [V1])."""
    return np.maximum(x, 0.0)


def sigmoid(x):
    """Output gate sigma(g) ([GBLA])."""
    return 1.0 / (1.0 + np.exp(-x))


# ----------------------------------------------------------------------- RoPE

def rope_pair_split(d):
    """Rotation pairs given to the (t, h, w) axes: see the module docstring."""
    assert d % 2 == 0 and d >= 2
    p = d // 2
    p_hw = p // 3
    return p - 2 * p_hw, p_hw, p_hw


def token_positions(T, H, W, t0=0):
    """(t, h, w) of every token in raster order n = (t*H + h)*W + w."""
    n = np.arange(T * H * W)
    t = n // (H * W) + t0
    h = (n // W) % H
    w = n % W
    return t, h, w


def rope_angles(d, T, H, W, rope_theta, t0=0):
    """Rotation angle of every (token, pair): array [N, d/2] ([V1] 3D RoPE)."""
    t, h, w = token_positions(T, H, W, t0)
    cols = []
    for pos, p in zip((t, h, w), rope_pair_split(d)):
        if p == 0:
            continue
        freq = rope_theta ** (-np.arange(p) / p)
        cols.append(pos[:, None].astype(np.float64) * freq[None, :])
    return np.concatenate(cols, axis=1)


def rope_rotate(x, angles):
    """Rotate channel pairs (2i, 2i+1) of x [B, N, Hh, d] by angles [N, d/2]."""
    c = np.cos(angles)[None, :, None, :]
    s = np.sin(angles)[None, :, None, :]
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def feature_maps(x, angles):
    """x -> (x_pls, x_til): RMSNorm, ReLU, then RoPE on the ReLU output
    ([GBLA] normalised q/k, [V1] RoPE(phi(x)))."""
    x_pls = relu(rms_normalize(x))
    x_til = x_pls if angles is None else rope_rotate(x_pls, angles)
    return x_pls, x_til


def _angles_or_none(d, T, H, W, rope_theta, t0):
    if rope_theta <= 0:
        return None
    return rope_angles(d, T, H, W, rope_theta, t0)


# ------------------------------------------------------- factorised operator

def state_and_keysum(k_til, k_pls, v, beta):
    """S[b,h] = sum_n v_n (beta_n k_til_n)^T  ([LA]);  z[b,h] = sum_n k_pls_n.

    Returns S [B, Hh, d, d] with S[..., a, c] = sum_n v_n[a] beta_n k_til_n[c],
    and z [B, Hh, d]."""
    B, N, Hh, d = v.shape
    S = np.empty((B, Hh, d, d))
    for b in range(B):
        for h in range(Hh):
            S[b, h] = v[b, :, h, :].T @ (beta[b, :, h, None] * k_til[b, :, h, :])
    z = k_pls.sum(axis=1)
    return S, z


def read_out(S, z, q_pls, q_til, g, eps):
    """den_j = z.q_pls_j + eps; pre_j = S q_til_j / den_j; x_j = sigma(g_j) pre_j;
    o_j = RMSNorm(x_j)  ([GBLA], denominator without RoPE per [V1])."""
    B, N, Hh, d = q_til.shape
    den = np.einsum("bnhc,bhc->bnh", q_pls, z) + eps
    u = np.empty_like(q_til)
    for b in range(B):
        for h in range(Hh):
            u[b, :, h, :] = q_til[b, :, h, :] @ S[b, h].T
    pre = u / den[..., None]
    x = sigmoid(g) * pre
    out = rms_normalize(x)
    return dict(den=den, pre=pre, x=x, out=out)


def forward(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=0):
    """Bidirectional operator over all N = T*H*W tokens, factorised form.

    Returns a dict with out, S, z, den, pre (S q_til / den) and x (gated,
    before the output norm)."""
    d = q.shape[-1]
    assert q.shape[1] == T * H * W
    angles = _angles_or_none(d, T, H, W, rope_theta, t0)
    q_pls, q_til = feature_maps(q, angles)
    k_pls, k_til = feature_maps(k, angles)
    S, z = state_and_keysum(k_til, k_pls, v, beta)
    res = read_out(S, z, q_pls, q_til, g, eps)
    res.update(S=S, z=z)
    return res


# -------------------------------------------------------- brute-force O(N^2)

def forward_bruteforce(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=0,
                       visible=None):
    """The operator written as a sum over token pairs, without forming S or z:

        pre_j = sum_n v_n beta_n (k_til_n . q_til_j)
                / (sum_n k_pls_n . q_pls_j + eps)

    visible(j, n) -> bool restricts the pairs (used for the block-causal
    mask); None means all pairs (bidirectional).  Python loops: tiny inputs
    only."""
    B, N, Hh, d = q.shape
    angles = _angles_or_none(d, T, H, W, rope_theta, t0)
    q_pls, q_til = feature_maps(q, angles)
    k_pls, k_til = feature_maps(k, angles)
    pre = np.zeros_like(q)
    for b in range(B):
        for h in range(Hh):
            for j in range(N):
                num = np.zeros(d)
                den = eps
                for n in range(N):
                    if visible is not None and not visible(j, n):
                        continue
                    num += v[b, n, h] * beta[b, n, h] * np.dot(k_til[b, n, h], q_til[b, j, h])
                    den += np.dot(k_pls[b, n, h], q_pls[b, j, h])
                pre[b, j, h] = num / den
    x = sigmoid(g) * pre
    return dict(pre=pre, x=x, out=rms_normalize(x))


# ------------------------------------------------------------- block-causal

def block_causal_step(S, z, q, k, v, beta, g, T_blk, H, W, t0, rope_theta, eps):
    """One block of the block-causal variant ([BLK]): add the block's own
    state and key sum to the carried (S, z), then read the block's tokens out
    against the updated (inclusive) state.  RoPE time = t0 + local frame.

    S [B, Hh, d, d] and z [B, Hh, d] are returned updated (new arrays)."""
    d = q.shape[-1]
    angles = _angles_or_none(d, T_blk, H, W, rope_theta, t0)
    q_pls, q_til = feature_maps(q, angles)
    k_pls, k_til = feature_maps(k, angles)
    dS, dz = state_and_keysum(k_til, k_pls, v, beta)
    S = S + dS
    z = z + dz
    res = read_out(S, z, q_pls, q_til, g, eps)
    res.update(S=S, z=z)
    return res


def block_causal_forward(q, k, v, beta, g, n_blocks, T_blk, H, W, rope_theta, eps):
    """Run block_causal_step over n_blocks consecutive blocks of T_blk*H*W
    tokens each, starting from S = 0, z = 0.  Returns out over all tokens and
    the final (S, z)."""
    B, N, Hh, d = q.shape
    L = T_blk * H * W
    assert N == n_blocks * L
    S = np.zeros((B, Hh, d, d))
    z = np.zeros((B, Hh, d))
    out = np.empty_like(q)
    for i in range(n_blocks):
        sl = slice(i * L, (i + 1) * L)
        r = block_causal_step(S, z, q[:, sl], k[:, sl], v[:, sl], beta[:, sl],
                              g[:, sl], T_blk, H, W, i * T_blk, rope_theta, eps)
        S, z = r["S"], r["z"]
        out[:, sl] = r["out"]
    return dict(out=out, S=S, z=z)


def block_causal_bruteforce(q, k, v, beta, g, n_blocks, T_blk, H, W, rope_theta, eps):
    """Prefix-masked brute force: token j sees token n iff block(n) <= block(j).
    Positions are those of the whole T = n_blocks*T_blk frame grid."""
    L = T_blk * H * W
    return forward_bruteforce(q, k, v, beta, g, n_blocks * T_blk, H, W, rope_theta,
                              eps, visible=lambda j, n: n // L <= j // L)


# -------------------------------------------------------- token-level causal

def causal_forward(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=0):
    """Token-level causal variant: token j is read out against the running
    sums, over tokens 0..j, of the per-token states v_n (beta_n k_til_n)^T and
    of the key features k_pls_n ([BLK]: causal linear attention needs only
    these two running sums; a token sees itself, as a block does).

        S_j = sum_{n<=j} v_n (beta_n k_til_n)^T      z_j = sum_{n<=j} k_pls_n
        den_j = z_j . q_pls_j + eps                  pre_j = S_j q_til_j / den_j

    Positions and the rest of the read-out as in forward().  The running sums
    are np.cumsum over the per-token terms, so memory grows as N*d*d: small
    inputs only."""
    d = q.shape[-1]
    assert q.shape[1] == T * H * W
    angles = _angles_or_none(d, T, H, W, rope_theta, t0)
    q_pls, q_til = feature_maps(q, angles)
    k_pls, k_til = feature_maps(k, angles)
    B, N, Hh, _ = q.shape
    den = np.empty((B, N, Hh))
    pre = np.empty_like(q)
    for b in range(B):
        for h in range(Hh):
            per_token = v[b, :, h, :, None] * (beta[b, :, h, None, None] * k_til[b, :, h, None, :])
            S_run = np.cumsum(per_token, axis=0)                  # [N, d, d]
            z_run = np.cumsum(k_pls[b, :, h, :], axis=0)          # [N, d]
            den[b, :, h] = np.einsum("nc,nc->n", z_run, q_pls[b, :, h, :]) + eps
            pre[b, :, h, :] = np.einsum("nac,nc->na", S_run, q_til[b, :, h, :]) / den[b, :, h, None]
    x = sigmoid(g) * pre
    return dict(den=den, pre=pre, x=x, out=rms_normalize(x))


def causal_forward_at(q, k, v, beta, g, T, H, W, rope_theta, eps, tokens, t0=0,
                      S0=None, z0=None):
    """The token-level causal read-out at the selected tokens only, each from
    its own prefix (the definition above, token by token, with no running
    sums):  S_j = S0 + sum_{n<=j} v_n (beta_n k_til_n)^T,
    z_j = z0 + sum_{n<=j} k_pls_n, and the read-out of token j against them.
    S0 [B, Hh, d, d] and z0 [B, Hh, d] are a state carried in from earlier
    tokens (zero if None), as a streaming call continues a sequence.  Memory
    stays O(N d), so it serves full-size inputs.  Returns den, pre, x, out of
    shape [B, len(tokens), Hh(, d)] and the state after the last token,
    S_end / z_end."""
    d = q.shape[-1]
    B, N, Hh, _ = q.shape
    assert N == T * H * W
    angles = _angles_or_none(d, T, H, W, rope_theta, t0)
    q_pls, q_til = feature_maps(q, angles)
    k_pls, k_til = feature_maps(k, angles)
    S0 = np.zeros((B, Hh, d, d)) if S0 is None else S0
    z0 = np.zeros((B, Hh, d)) if z0 is None else z0
    tokens = list(tokens)
    den = np.empty((B, len(tokens), Hh))
    u = np.empty((B, len(tokens), Hh, d))
    for i, j in enumerate(tokens):
        S, z = state_and_keysum(k_til[:, :j + 1], k_pls[:, :j + 1], v[:, :j + 1],
                                beta[:, :j + 1])
        r = read_out(S0 + S, z0 + z, q_pls[:, j:j + 1], q_til[:, j:j + 1], g[:, j:j + 1], eps)
        den[:, i] = r["den"][:, 0]
        u[:, i] = r["pre"][:, 0]
    x = sigmoid(g[:, tokens]) * u
    S, z = state_and_keysum(k_til, k_pls, v, beta)
    return dict(den=den, pre=u, x=x, out=rms_normalize(x), S_end=S0 + S, z_end=z0 + z)


def causal_bruteforce(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=0):
    """Prefix-masked pair sum: token j sees token n iff n <= j."""
    return forward_bruteforce(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=t0,
                              visible=lambda j, n: n <= j)


# ------------------------------------------------- MXFP8 operator inputs

# The MX block formats (OCP Microscaling): elements in FP8 E4M3, one shared
# E8M0 power-of-two scale per MX_BLOCK consecutive elements along the
# innermost axis (the head dim here).  Reading for the FP8-input row: q, k, v
# and g arrive in this format, beta stays in its own dtype, and the operator
# is the one above applied to the decoded values.

MX_BLOCK = 32


def e4m3_decode(codes):
    """FP8 E4M3 without infinities: sign bit, 4 exponent bits (bias 7), 3
    mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6, and
    S.1111.111 is NaN (the largest finite value is 1.75 * 2^8 = 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    out = sign * mag
    out[(e == 15) & (c & 0x7 == 7)] = np.nan
    return out


def e8m0_decode(codes):
    """E8M0 scale: 2^(code - 127); code 255 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.float64)
    out = np.exp2(c - 127.0)
    out[c == 255] = np.nan
    return out


def mx_dequantize(codes, scales):
    """Element i of a row is e4m3(codes[..., i]) * e8m0(scales[..., i // MX_BLOCK])."""
    x = e4m3_decode(codes)
    sc = e8m0_decode(scales)
    assert sc.shape[-1] * MX_BLOCK == x.shape[-1]
    return x * np.repeat(sc, MX_BLOCK, axis=-1)


def forward_mx(q, k, v, beta, g, T, H, W, rope_theta, eps, t0=0):
    """The bidirectional operator on MX inputs: q, k, v and g are (codes,
    scales) pairs, beta a float array."""
    dq = lambda pair: mx_dequantize(*pair)
    return forward(dq(q), dq(k), dq(v), beta, dq(g), T, H, W, rope_theta, eps, t0)


# ------------------------------------------------------ gated softmax anchor

def softmax_anchor(q, k, v, g, T, H, W, rope_theta, t0=0, queries=None):
    """The gated softmax anchor of the hybrid stack ([GBLA]'s page, "softmax
    anchors and hybrid attention"; method: a gated softmax layer every fourth
    depth): bidirectional scaled dot-product attention with QK normalisation,
    RoPE and a sigmoid output gate.  Readings: RMSNorm per head over d (no
    weight, epsilon RMS_EPS), the library's 3D RoPE spec on the normalised q
    and k (no ReLU on this path), scores q_til . k_til / sqrt(d) over every
    token, and o_j = sigmoid(g_j) * sum_n softmax_n(scores_j) v_n, with no
    output norm (W_o is outside).  q, k, v, g [B, N, Hh, d]; returns dict(out,
    attn) with attn the read-out before the gate.  queries: indices of the
    query tokens whose rows are returned ([B, len(queries), Hh, d]); default
    all tokens."""
    d = q.shape[-1]
    angles = _angles_or_none(d, T, H, W, rope_theta, t0)
    qh, kh = rms_normalize(q), rms_normalize(k)
    qt = qh if angles is None else rope_rotate(qh, angles)
    kt = kh if angles is None else rope_rotate(kh, angles)
    B, N, Hh, _ = q.shape
    rows = np.arange(N) if queries is None else np.asarray(queries)
    attn = np.empty((B, len(rows), Hh, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hh):
            s = qt[b, rows, h, :] @ kt[b, :, h, :].T / np.sqrt(d)
            s = s - s.max(axis=1, keepdims=True)
            w = np.exp(s)
            w /= w.sum(axis=1, keepdims=True)
            attn[b, :, h, :] = w @ v[b, :, h, :]
    return dict(attn=attn, out=sigmoid(g[:, rows]) * attn)


# ----------------------------------------------- the layer's projections

# [GBLA] writes the read-out as o_j = W_o RMSNorm[...]: the heads' normalised
# read-outs, concatenated over the heads (the width Hh*d), times W_o.  The
# pages print no input projection; reading: q, k, v, g and the beta logits
# are one linear map of the layer input x (rows of W_in in that order: Hh*d
# rows each for q, k, v and g, then Hh rows of beta logits), with beta =
# sigmoid(logits) and g left as logits (the operator applies its sigmoid).

def project_in(x, W_in, heads, head_dim):
    """x [B, N, C], W_in [4*Hh*d + Hh, C] -> dict(q, k, v, g [B, N, Hh, d],
    beta [B, N, Hh]) with beta = sigmoid(x W_beta^T)."""
    B, N, _ = x.shape
    hd = heads * head_dim
    y = x @ W_in.T
    out = {}
    for i, name in enumerate("qkvg"):
        out[name] = y[..., i * hd:(i + 1) * hd].reshape(B, N, heads, head_dim)
    out["beta"] = sigmoid(y[..., 4 * hd:4 * hd + heads])
    return out


def project_out(o, W_o):
    """o [B, N, Hh, d] (the operator's output) -> o_flat W_o^T, [B, N, C_out]
    with W_o [C_out, Hh*d]."""
    B, N, Hh, d = o.shape
    return o.reshape(B, N, Hh * d) @ W_o.T


def layer_forward(x, W_in, W_o, heads, head_dim, T, H, W, rope_theta, eps):
    """x -> projections -> the bidirectional operator -> W_o."""
    p = project_in(x, W_in, heads, head_dim)
    r = forward(p["q"], p["k"], p["v"], p["beta"], p["g"], T, H, W, rope_theta, eps)
    return dict(y=project_out(r["out"], W_o), proj=p, op=r)


# ------------------------------------------------------------- parity metric

def max_err_over_rms(got, ref):
    """max_i |got_i - ref_i| / rms(ref)  (the bf16 tolerance metric)."""
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref)) / rms)


def max_rel_err_rms_floor(got, ref):
    """max_i |got_i - ref_i| / max(|ref_i|, rms(ref))  (the fp32 metric:
    relative for elements at or above the RMS, RMS-relative below it)."""
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), rms)))


def bf16_half_ulp(ref):
    """Half the spacing of bf16 numbers (8 significant bits) at |ref|: the
    largest error of a correctly rounded bf16 result."""
    a = np.maximum(np.abs(np.asarray(ref, dtype=np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, (np.floor(np.log2(a)) - 8).astype(int))


def bf16_out_err_over_rms(got, ref):
    """Error of a bf16 output beyond its own rounding, over rms(ref):
    max_i max(0, |got_i - ref_i| - bf16_half_ulp(ref_i)) / rms(ref).  A
    correctly rounded result of the exact value scores 0; the rounding alone
    reaches 1.56e-2 x rms for outputs in [4, 8) and is not arithmetic error."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    excess = np.maximum(np.abs(got - ref) - bf16_half_ulp(ref), 0.0)
    return float(np.max(excess) / np.sqrt(np.mean(ref * ref)))


def max_err_over_row_rms(got, ref):
    """max over rows r and elements i of |got_ri - ref_ri| / rms(ref_r), rows
    being the last axis (a token's d channels): the error relative to each
    token's own RMS.  The causal read-out's pre-norm values differ in scale
    from token to token (an early token averages few values), so its
    tolerance is stated per token, as the output's is after its RMSNorm."""
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    return float(np.max(np.abs(got - ref) / rms))
