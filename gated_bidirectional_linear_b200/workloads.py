"""Seeded synthetic workloads shaped like SANA-Video latent-video attention layers.

This module only draws inputs.  It holds none of the operator's arithmetic, so
both the CUDA library's tests/bench and the CPU oracle take their inputs from
here without sharing any of the method.

Recipe (every config): numpy PCG64 seeded with the config's seed; draw, in this
order, q, k, v, g ~ N(0, 1) and then the beta logits ~ N(0, 1), each of shape
[B, N, Hh, d] (logits [B, N, Hh]); beta = logistic(logits); everything is then
rounded (round-to-nearest-even) to the config's dtype.  The rounded values are
the inputs of both sides.

Shapes (latent grids of the SANA-Video pages: 480x832x81 -> 11x15x26 tokens,
736x1280x121 -> 16x23x40; widths 2560 = 20x128 and 4096 = 32x128 for the 5B
and 14B models).
"""
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    dtype: str              # "f32" or "bf16"
    seed: int
    rope_theta: float = 10000.0
    eps: float = 1e-6
    n_blocks: int = 1       # >1: block-causal, T is the frames of ONE block

    @property
    def tokens(self):
        """Tokens per call (one block for the block-causal variant)."""
        return self.T * self.H * self.W

    @property
    def total_tokens(self):
        return self.tokens * self.n_blocks

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self):
        return 4 if self.dtype == "f32" else 2

    def alg_bytes_per_call(self):
        """q, k, v, g read + out written (5 [B,N,Hh,d] tensors) + beta read."""
        th = self.batch * self.tokens * self.heads
        return th * (5 * self.head_dim + 1) * self.elem_bytes

    def flops_per_call(self):
        """2d^2 for the state contraction + 2d^2 for the read-out, per token-head."""
        th = self.batch * self.tokens * self.heads
        return th * 4 * self.head_dim * self.head_dim


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 32, 2, 4, 4, "f32", seed=0),
    "480p": Workload("480p", 1, 20, 128, 11, 15, 26, "bf16", seed=1),
    "720p": Workload("720p", 2, 20, 128, 16, 23, 40, "bf16", seed=2),
    "14b": Workload("14b", 1, 32, 128, 61, 23, 40, "bf16", seed=3),
    "blk": Workload("blk", 1, 20, 128, 3, 23, 40, "bf16", seed=4, n_blocks=20),
}


def _round(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.float32 if dtype == "f32" else torch.bfloat16)


def draw(batch, tokens, heads, head_dim, dtype, seed):
    """Seeded inputs as CPU torch tensors in `dtype` ("f32" or "bf16").

    Returns dict(q, k, v, g, beta) with q..g [B, N, Hh, d] and beta [B, N, Hh]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = (batch, tokens, heads, head_dim)
    out = {}
    for name in ("q", "k", "v", "g"):
        out[name] = _round(rng.standard_normal(shape, dtype=np.float32), dtype)
    logits = rng.standard_normal(shape[:3], dtype=np.float64)
    out["beta"] = _round((1.0 / (1.0 + np.exp(-logits))).astype(np.float32), dtype)
    return out


MX_BLOCK = 32          # elements per shared scale (OCP MX)
E4M3_EMAX = 8          # exponent of E4M3's largest power of two (448 = 1.75 * 2^8)


def mx_encode(x):
    """OCP MX encoding of a float array along its last axis, as the inputs of
    the FP8 operator arrive: per block of 32 consecutive elements one E8M0
    shared exponent X = floor(log2(max |x|)) - 8 (biased by 127; a block of
    zeros takes the smallest), elements x / 2^X rounded to nearest-even E4M3
    and clamped to +-448.  Returns (codes uint8 [..., d], scales uint8
    [..., d/32]) as CPU torch tensors."""
    x = np.asarray(x, dtype=np.float32)
    d = x.shape[-1]
    blocks = x.reshape(x.shape[:-1] + (d // MX_BLOCK, MX_BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    with np.errstate(divide="ignore"):
        e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))), -127.0)
    X = np.clip(e - E4M3_EMAX, -127, 127)
    elems = np.clip(blocks / np.exp2(X)[..., None], -448.0, 448.0).astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(elems.reshape(x.shape))).to(
        torch.float8_e4m3fn).view(torch.uint8)
    scales = torch.from_numpy((X + 127).astype(np.uint8))
    return codes, scales


def draw_mx(batch, tokens, heads, head_dim, seed):
    """Seeded MX inputs: the same draws as draw() (q, k, v, g ~ N(0, 1), beta
    = logistic(N(0, 1))) with q, k, v and g MX-encoded and beta in bf16.
    Returns dict(q, q_scale, k, k_scale, v, v_scale, g, g_scale, beta)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = (batch, tokens, heads, head_dim)
    out = {}
    for name in ("q", "k", "v", "g"):
        out[name], out[name + "_scale"] = mx_encode(rng.standard_normal(shape, dtype=np.float32))
    logits = rng.standard_normal(shape[:3], dtype=np.float64)
    out["beta"] = _round((1.0 / (1.0 + np.exp(-logits))).astype(np.float32), "bf16")
    return out


def make_inputs(wl: Workload, seed=None):
    """Inputs of a workload over all of its tokens (all blocks)."""
    return draw(wl.batch, wl.total_tokens, wl.heads, wl.head_dim, wl.dtype,
                wl.seed if seed is None else seed)


def as_f64(inputs):
    """The same inputs as float64 numpy arrays (exact: both dtypes embed)."""
    return {k: v.to(torch.float64).numpy() for k, v in inputs.items()}
