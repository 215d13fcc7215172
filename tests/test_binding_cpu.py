"""The Python binding's argument checks (CPU only).

The C ABI receives raw pointers and cannot see a tensor's shape, dtype,
strides or device; the binding checks those before anything is launched, so
a mismatched call raises ValueError instead of reading the wrong memory."""
import pytest
import torch

from gated_bidirectional_linear_b200 import gla

T, H, W, B, HEADS, D = 2, 3, 4, 1, 2, 128


def host_inputs(dtype=torch.bfloat16):
    n = T * H * W
    x = {k: torch.zeros(B, n, HEADS, D, dtype=dtype) for k in ("q", "k", "v", "g")}
    x["beta"] = torch.zeros(B, n, HEADS, dtype=dtype)
    return x


def call_host(x, **kw):
    return gla.gla_forward_host(x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W, **kw)


def test_device_entry_rejects_host_tensors():
    x = host_inputs()
    with pytest.raises(ValueError, match="GPU"):
        gla.gla_forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W)
    with pytest.raises(ValueError, match="GPU"):
        gla.gla_forward_noalloc(x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W)
    S = torch.zeros(B, HEADS, D, D)
    z = torch.zeros(B, HEADS, D)
    with pytest.raises(ValueError, match="GPU"):
        gla.gla_block_causal_step(S, z, x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W, 0)


def test_grid_must_match_tokens():
    x = host_inputs()
    with pytest.raises(ValueError, match="tokens"):
        gla.gla_forward_host(x["q"], x["k"], x["v"], x["beta"], x["g"], T + 1, H, W)


@pytest.mark.parametrize("name,bad", [
    ("k", lambda t: t[:, :, :1].clone()),                 # wrong shape
    ("v", lambda t: t.transpose(2, 3)),                   # wrong shape (transposed)
    ("g", lambda t: t.float()),                           # wrong dtype
    ("beta", lambda t: t.unsqueeze(-1).clone()),          # wrong rank
    ("v", lambda t: torch.zeros(t.shape[0], t.shape[1], t.shape[3], t.shape[2],
                                dtype=t.dtype).transpose(2, 3)),   # right shape, not contiguous
])
def test_mismatched_inputs_raise(name, bad):
    x = host_inputs()
    x[name] = bad(x[name])
    with pytest.raises(ValueError, match=name):
        call_host(x)


def test_out_must_match():
    x = host_inputs()
    with pytest.raises(ValueError, match="out"):
        call_host(x, out=torch.zeros(B, T * H * W, HEADS, D, dtype=torch.float32))


def test_host_entry_rejects_host_arena():
    x = host_inputs()
    with pytest.raises(ValueError, match="arena"):
        call_host(x, arena=torch.zeros(1 << 20, dtype=torch.uint8))


class _FakeStream:
    def __init__(self, device):
        self.device = torch.device(device)
        self.cuda_stream = 0


def test_stream_of_another_device_is_refused():
    """The library launches on the current device, which the binding sets to
    the tensors' device for each call; a stream of a different device would
    put the kernels on one GPU and the pointers on another."""
    with pytest.raises(ValueError, match="stream"):
        gla._stream(_FakeStream("cuda:1"), torch.device("cuda", 0))
    assert gla._stream(_FakeStream("cuda:0"), torch.device("cuda", 0)).value in (None, 0)


def test_other_entries_reject_host_tensors():
    x = host_inputs()
    S = torch.zeros(B, HEADS, D, D)
    z = torch.zeros(B, HEADS, D)
    with pytest.raises(ValueError, match="GPU"):
        gla.gla_causal_step(S, z, x["q"], x["k"], x["v"], x["beta"], x["g"], T, H, W)
    with pytest.raises(ValueError, match="GPU"):
        gla.gla_softmax_anchor(x["q"], x["k"], x["v"], x["g"], T, H, W)
    a = torch.zeros(16, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="GPU"):
        gla.gla_gemm_bf16(a, a)
    mx = {n: torch.zeros(B, T * H * W, HEADS, D, dtype=torch.uint8) for n in "qkvg"}
    mx.update({n + "_scale": torch.zeros(B, T * H * W, HEADS, 4, dtype=torch.uint8) for n in "qkvg"})
    mx["beta"] = x["beta"]
    with pytest.raises(ValueError):
        gla.gla_forward_mx(mx, T, H, W)


def test_anchor_checks_dtype_and_shape():
    x = host_inputs()
    with pytest.raises(ValueError, match="v"):
        gla.gla_softmax_anchor(x["q"], x["k"], x["v"].float(), x["g"], T, H, W)
    with pytest.raises(ValueError, match="tokens"):
        gla.gla_softmax_anchor(x["q"], x["k"], x["v"], x["g"], T + 1, H, W)
