"""Guard bands around every buffer the library writes (compute-sanitizer is
not available, so out-of-bounds writes are looked for directly): the output,
the workspace and the block-causal state sit inside larger allocations whose
margins hold a sentinel pattern, and the margins must come back untouched.
Shapes are ragged (a partial last tile, heads that straddle CTAs)."""
import pytest
import torch

from gated_bidirectional_linear_b200 import gla, workloads
from gpu_common import to_device

pytestmark = pytest.mark.gpu

GUARD = 8192            # elements of margin on each side (16-byte multiples)
SENT16 = 0x7FC1         # a NaN pattern no result takes
SENT8 = 0xA5


def guarded(shape, dtype):
    """A tensor of `shape` inside a flat buffer with GUARD elements of
    sentinel on both sides; returns (view, buffer)."""
    n = 1
    for s in shape:
        n *= s
    buf = torch.empty(GUARD + n + GUARD, dtype=dtype, device="cuda")
    if dtype == torch.bfloat16:
        buf.view(torch.int16).fill_(SENT16)
    elif dtype == torch.uint8:
        buf.fill_(SENT8)
    else:
        buf.view(torch.int32).fill_(0x7FC00001)
    return buf[GUARD:GUARD + n].view(shape), buf


def margins_intact(buf, n):
    head, tail = buf[:GUARD], buf[GUARD + n:]
    if buf.dtype == torch.bfloat16:
        return bool((head.view(torch.int16) == SENT16).all() and
                    (tail.view(torch.int16) == SENT16).all())
    if buf.dtype == torch.uint8:
        return bool((head == SENT8).all() and (tail == SENT8).all())
    return bool((head.view(torch.int32) == 0x7FC00001).all() and
                (tail.view(torch.int32) == 0x7FC00001).all())


@pytest.mark.parametrize("path", [gla.GLA_PATH_TENSOR, gla.GLA_PATH_SIMT], ids=["tensor", "simt"])
def test_forward_writes_stay_inside(path):
    B, HH, T, H, W = 2, 3, 3, 7, 9          # N = 189: one full 128-token tile and a ragged one
    N = T * H * W
    d = to_device(workloads.draw(B, N, HH, 128, "bf16", seed=41))
    out, obuf = guarded((B, N, HH, 128), torch.bfloat16)
    nws = gla.gla_forward_workspace_size(B, HH, 128, T, H, W, gla.GLA_DTYPE_BF16)
    ws, wbuf = guarded((nws,), torch.uint8)
    gla.gla_forward(d["q"], d["k"], d["v"], d["beta"], d["g"], T, H, W, out=out, workspace=ws,
                    path=path)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    assert margins_intact(obuf, out.numel()), "write outside out"
    assert margins_intact(wbuf, nws), "write outside the workspace"
    assert not torch.isnan(out.float()).any(), "output element left unwritten"


def test_block_causal_writes_stay_inside():
    B, HH, T, H, W = 1, 5, 2, 5, 11          # N = 110 per block: a ragged single tile
    N = T * H * W
    d = to_device(workloads.draw(B, N, HH, 128, "bf16", seed=43))
    S, sbuf = guarded((B, HH, 128, 128), torch.float32)
    z, zbuf = guarded((B, HH, 128), torch.float32)
    S.zero_()
    z.zero_()
    out, obuf = guarded((B, N, HH, 128), torch.bfloat16)
    nws = gla.gla_block_causal_workspace_size(B, HH, 128, T, H, W, gla.GLA_DTYPE_BF16)
    ws, wbuf = guarded((nws,), torch.uint8)
    for step in range(2):
        gla.gla_block_causal_step(S, z, d["q"], d["k"], d["v"], d["beta"], d["g"], T, H, W,
                                  step * T, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    for name, buf, n in (("state", sbuf, S.numel()), ("z", zbuf, z.numel()),
                         ("out", obuf, out.numel()), ("workspace", wbuf, nws)):
        assert margins_intact(buf, n), f"write outside {name}"
