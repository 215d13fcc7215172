"""The entry points beyond gla_forward reject bad arguments on the host,
before any device call: token-level causal, FP8 (MX) inputs, the layer's
GEMMs and the gated softmax anchor.  No GPU needed: the pointers are never
dereferenced."""
import pytest

from gated_bidirectional_linear_b200 import gla

FAKE = 1 << 20          # a 16-byte aligned address that is never dereferenced
OK_SIZE = 1 << 30


def _causal(**kw):
    a = dict(S=FAKE, z=FAKE, q=FAKE, k=FAKE, v=FAKE, beta=FAKE, g=FAKE, B=1, Hh=2, d=128, T=2,
             H=4, W=4, t0=0, theta=1e4, eps=1e-6, dtype=gla.GLA_DTYPE_BF16, out=FAKE, ws=FAKE,
             wsb=OK_SIZE, stream=None, path=gla.GLA_PATH_AUTO)
    a.update(kw)
    return gla.lib().gla_causal_step_ex(*a.values(), None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(S=None), gla.GLA_ERR_INVALID_ARG),
    (dict(z=FAKE + 4), gla.GLA_ERR_INVALID_ARG),            # misaligned
    (dict(t0=-1), gla.GLA_ERR_INVALID_ARG),
    (dict(eps=0.0), gla.GLA_ERR_INVALID_ARG),
    (dict(theta=float("inf")), gla.GLA_ERR_INVALID_ARG),
    (dict(d=48), gla.GLA_ERR_INVALID_ARG),
    (dict(path=9), gla.GLA_ERR_UNSUPPORTED),
    (dict(dtype=gla.GLA_DTYPE_F32, path=gla.GLA_PATH_TENSOR), gla.GLA_ERR_UNSUPPORTED),
])
def test_causal_rejects(kw, status):
    assert _causal(**kw) == status


def _mx(**kw):
    a = dict(q=FAKE, qs=FAKE, k=FAKE, ks=FAKE, v=FAKE, vs=FAKE, beta=FAKE, g=FAKE, gs=FAKE, B=1,
             Hh=2, d=128, T=2, H=4, W=4, theta=1e4, eps=1e-6, out=FAKE, ws=FAKE, wsb=OK_SIZE,
             stream=None, path=gla.GLA_PATH_AUTO)
    a.update(kw)
    return gla.lib().gla_forward_mx_ex(*a.values(), None, None, None, None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(ks=None), gla.GLA_ERR_INVALID_ARG),
    (dict(gs=FAKE + 8), gla.GLA_ERR_INVALID_ARG),
    (dict(d=64), gla.GLA_ERR_UNSUPPORTED),                    # the MX kernels take d = 128
    (dict(eps=-1.0), gla.GLA_ERR_INVALID_ARG),
    (dict(path=5), gla.GLA_ERR_UNSUPPORTED),
    (dict(ws=None), gla.GLA_ERR_WORKSPACE),
    (dict(ws=FAKE + 16), gla.GLA_ERR_WORKSPACE),
])
def test_mx_rejects(kw, status):
    assert _mx(**kw) == status


@pytest.mark.parametrize("M,N,K,status", [
    (0, 8, 8, gla.GLA_ERR_INVALID_ARG),
    (8, 12, 8, gla.GLA_ERR_INVALID_ARG),      # N not a multiple of 8
    (8, 8, 20, gla.GLA_ERR_INVALID_ARG),      # K not a multiple of 8
])
def test_gemm_rejects(M, N, K, status):
    assert gla.lib().gla_gemm_bf16(FAKE, FAKE, FAKE, M, N, K, None) == status


def test_gemm_rejects_misaligned():
    assert gla.lib().gla_gemm_bf16(FAKE + 2, FAKE, FAKE, 8, 8, 8, None) == gla.GLA_ERR_INVALID_ARG


def test_project_in_rejects():
    lib = gla.lib()
    P = [FAKE] * 5
    assert lib.gla_project_in(FAKE, FAKE, 16, 12, 2, 128, *P, None) == gla.GLA_ERR_INVALID_ARG
    assert lib.gla_project_in(FAKE, FAKE, 16, 16, 1, 16, *P, None) == gla.GLA_ERR_UNSUPPORTED
    assert lib.gla_project_in(FAKE, FAKE, 16, 16, 2, 128, FAKE, None, FAKE, FAKE, FAKE,
                              None) == gla.GLA_ERR_INVALID_ARG


def test_layer_rejects():
    lib = gla.lib()
    args = lambda C, C_out, ws, wsb: (FAKE, FAKE, FAKE, 1, C, C_out, 2, 128, 2, 4, 4, 1e4, 1e-6,
                                      FAKE, ws, wsb, None)
    assert lib.gla_layer_forward(*args(260, 256, FAKE, OK_SIZE)) == gla.GLA_ERR_UNSUPPORTED
    assert lib.gla_layer_forward(*args(256, 256, None, OK_SIZE)) == gla.GLA_ERR_WORKSPACE
    assert lib.gla_layer_forward(*args(256, 256, FAKE, 1024)) == gla.GLA_ERR_WORKSPACE
    assert lib.gla_layer_workspace_size(1, 2, 48, 2, 4, 4) == 0


def _anchor(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, B=1, Hh=2, d=128, T=2, H=4, W=4, theta=1e4,
             out=FAKE, ws=FAKE, wsb=OK_SIZE, stream=None)
    a.update(kw)
    return gla.lib().gla_softmax_anchor(*a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(v=None), gla.GLA_ERR_INVALID_ARG),
    (dict(out=FAKE + 2), gla.GLA_ERR_INVALID_ARG),
    (dict(T=0), gla.GLA_ERR_INVALID_ARG),
    (dict(theta=float("nan")), gla.GLA_ERR_INVALID_ARG),
    (dict(d=64), gla.GLA_ERR_UNSUPPORTED),
    (dict(B=256, Hh=256), gla.GLA_ERR_UNSUPPORTED),         # batch * heads over one grid axis
    (dict(ws=None), gla.GLA_ERR_WORKSPACE),
    (dict(ws=FAKE + 64), gla.GLA_ERR_WORKSPACE),
    (dict(wsb=1024), gla.GLA_ERR_WORKSPACE),
])
def test_anchor_rejects(kw, status):
    assert _anchor(**kw) == status


def test_anchor_workspace_size():
    # q_til and k_til, fp16, the inputs' layout, each rounded up to 256 bytes
    n = 2 * 14720 * 20 * 128 * 2
    assert gla.gla_softmax_anchor_workspace_size(2, 20, 128, 16, 23, 40) == 2 * n
    assert gla.gla_softmax_anchor_workspace_size(2, 20, 64, 16, 23, 40) == 0
