"""Block-causal state as a checkpoint, and the invariants that tie the
block-causal steps to the bidirectional call (GPU, tensor path).

- Checkpoint and resume: the carried (S, z) is the whole resumable state, so
  20 steps in one go and 10 steps, a round trip of (S, z) through host
  memory, then 10 more steps give bitwise equal outputs and states.
- After the last step the carried state is the full sequence's state: S and z
  equal those of one bidirectional gla_forward over all blocks (the sums differ
  only in their grouping), and the last block's output equals that call's
  output for those tokens.
- Output norm: every output row has RMS sqrt(ms / (ms + 1e-6)), ms the mean
  square of the row before the norm, up to the bf16 rounding."""
import numpy as np
import pytest
import torch

from gated_bidirectional_linear_b200 import gla, workloads
from gpu_common import BF16_TOL, S_TOL_BF16, ZDEN_TOL, bf16_half_ulp, np64, rel_elem, rel_floor

pytestmark = pytest.mark.gpu


def _steps(d, wl, state, z, first, count, ws):
    L = wl.tokens
    outs = []
    for i in range(first, first + count):
        sl = slice(i * L, (i + 1) * L)
        blk = {k: v[:, sl].contiguous() for k, v in d.items()}
        outs.append(gla.gla_block_causal_step(state, z, blk["q"], blk["k"], blk["v"], blk["beta"],
                                              blk["g"], wl.T, wl.H, wl.W, i * wl.T, wl.rope_theta,
                                              wl.eps, workspace=ws))
    return outs


@pytest.fixture(scope="module")
def blk():
    wl = workloads.WORKLOADS["blk"]
    inp = workloads.make_inputs(wl)
    d = {k: v.cuda() for k, v in inp.items()}
    B, N, Hh, hd = d["q"].shape
    ws = gla.alloc_workspace(gla.gla_block_causal_workspace_size(
        B, Hh, hd, wl.T, wl.H, wl.W, gla.GLA_DTYPE_BF16))
    return wl, d, ws


def test_checkpoint_resume_is_bitwise(blk):
    wl, d, ws = blk
    B, N, Hh, hd = d["q"].shape
    torch.cuda.set_device(0)
    s1 = torch.zeros(B, Hh, hd, hd, device="cuda")
    z1 = torch.zeros(B, Hh, hd, device="cuda")
    straight = _steps(d, wl, s1, z1, 0, wl.n_blocks, ws)
    s2 = torch.zeros_like(s1)
    z2 = torch.zeros_like(z1)
    first = _steps(d, wl, s2, z2, 0, wl.n_blocks // 2, ws)
    torch.cuda.synchronize()
    s_host, z_host = s2.cpu().clone(), z2.cpu().clone()      # checkpoint
    s3, z3 = s_host.cuda(), z_host.cuda()                      # resume
    second = _steps(d, wl, s3, z3, wl.n_blocks // 2, wl.n_blocks - wl.n_blocks // 2, ws)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    for a, b in zip(straight, first + second):
        assert torch.equal(a, b)
    assert torch.equal(s1, s3) and torch.equal(z1, z3)


def test_last_block_state_equals_bidirectional_state(blk):
    wl, d, ws = blk
    B, N, Hh, hd = d["q"].shape
    s = torch.zeros(B, Hh, hd, hd, device="cuda")
    z = torch.zeros(B, Hh, hd, device="cuda")
    outs = _steps(d, wl, s, z, 0, wl.n_blocks, ws)
    T_all = wl.T * wl.n_blocks
    full = gla.gla_forward_debug(d["q"], d["k"], d["v"], d["beta"], d["g"], T_all, wl.H, wl.W,
                                 wl.rope_theta, wl.eps)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    assert rel_floor(np64(s), np64(full["S"])) <= S_TOL_BF16
    assert rel_elem(np64(z), np64(full["z"])) <= ZDEN_TOL
    last = np64(outs[-1])
    ref = np64(full["out"])[:, (wl.n_blocks - 1) * wl.tokens:]
    # Both sides are rounded to bf16 on their own, so an element may differ by
    # one bf16 spacing; the bar applies to what lies beyond that.
    excess = np.maximum(np.abs(last - ref) - 2 * bf16_half_ulp(ref), 0.0)
    assert excess.max() / np.sqrt(np.mean(ref * ref)) <= BF16_TOL


def test_output_rows_have_unit_rms():
    wl = workloads.WORKLOADS["480p"]
    d = {k: v.cuda() for k, v in workloads.make_inputs(wl).items()}
    r = gla.gla_forward_debug(d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W,
                              wl.rope_theta, wl.eps)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    x = np64(r["x"])
    ms = (x * x).mean(-1)
    expect = np.sqrt(ms / (ms + 1e-6))
    rms = np.sqrt((np64(r["out"]) ** 2).mean(-1))
    # Rounding to bf16 (8 significant bits) moves each element, and so a row's
    # RMS, by at most 2^-8 relative.
    assert np.all(np.abs(rms - expect) <= 2.0 ** -8 * expect + 1e-5), np.abs(rms - expect).max()


def test_host_step_entry_matches_device_steps():
    """gla_block_causal_step_host (host inputs and output, device-resident
    state) gives the device entry's outputs and state bit for bit, over three
    consecutive blocks."""
    T, H, W, B, HH, n = 2, 5, 9, 1, 3, 3
    L = T * H * W
    inp = workloads.draw(B, n * L, HH, 128, "bf16", seed=41)
    blocks = [{k: v[:, i * L:(i + 1) * L].contiguous() for k, v in inp.items()} for i in range(n)]
    S_d = torch.zeros(B, HH, 128, 128, device="cuda")
    z_d = torch.zeros(B, HH, 128, device="cuda")
    S_h, z_h = S_d.clone(), z_d.clone()
    for i, blk in enumerate(blocks):
        d = {k: v.cuda() for k, v in blk.items()}
        o_d = gla.gla_block_causal_step(S_d, z_d, d["q"], d["k"], d["v"], d["beta"], d["g"],
                                        T, H, W, i * T)
        p = {k: v.pin_memory() for k, v in blk.items()}
        o_h = torch.empty_like(p["q"]).pin_memory()
        gla.gla_block_causal_step_host(S_h, z_h, p["q"], p["k"], p["v"], p["beta"], p["g"],
                                       T, H, W, i * T, out=o_h)
        torch.cuda.synchronize()
        assert gla.gla_get_device_status() == gla.GLA_OK
        assert torch.equal(o_h, o_d.cpu())
    assert torch.equal(S_h, S_d) and torch.equal(z_h, z_d)
