"""The layer around the operator: the tcgen05 bf16 GEMM, the input projection
that writes the operator's inputs straight from its epilogue, and the whole
layer (projection, operator, W_o), against the fp64 oracle (numpy products of
the same bf16 values, oracle.project_in / project_out / layer_forward)."""
import numpy as np
import pytest
import torch

import oracle.gla_oracle as O
from gated_bidirectional_linear_b200 import gla, workloads
from gpu_common import BF16_TOL, np64, rel_rms, rel_rms_bf16out

pytestmark = pytest.mark.gpu


def _bf16(shape, seed, scale=1.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    return torch.from_numpy((rng.standard_normal(shape, dtype=np.float32) * scale)).to(
        torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 264, 200), (1, 8, 8), (4290, 2560, 2560),
                                   (1000, 520, 1032)])
def test_gemm_matches_fp64_products(M, N, K):
    A, B = _bf16((M, K), 1), _bf16((N, K), 2)
    C = gla.gla_gemm_bf16(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    ref = A.double().numpy() @ B.double().numpy().T
    err = rel_rms_bf16out(np64(C), ref)
    print(f"gemm {M}x{N}x{K}: {err:.2e} beyond bf16 rounding")
    assert err <= 1e-4


def test_project_in_writes_the_operator_inputs():
    B, T, H, W, Hh, d, C = 2, 2, 5, 7, 4, 128, 264
    N = T * H * W
    x = _bf16((B * N, C), 3)
    W_in = _bf16((4 * Hh * d + Hh, C), 4, scale=C ** -0.5)
    got = gla.gla_project_in(x.cuda(), W_in.cuda(), B, N, Hh, d)
    torch.cuda.synchronize()
    ref = O.project_in(x.double().numpy().reshape(B, N, C), W_in.double().numpy(), Hh, d)
    for name in ("q", "k", "v", "g", "beta"):
        err = rel_rms_bf16out(np64(got[name]), ref[name])
        assert err <= 1e-4, (name, err)


def test_layer_480p_shape():
    """The 5B width (2560 = 20 x 128) at the 480p grid: y against the fp64
    composition of the same bf16 x, W_in and W_o (the oracle does not round
    the intermediates the layer keeps in bf16, which the bar covers)."""
    wl = workloads.WORKLOADS["480p"]
    Hh, d, C = wl.heads, wl.head_dim, wl.heads * wl.head_dim
    N = wl.tokens
    x = _bf16((N, C), 5)
    W_in = _bf16((4 * Hh * d + Hh, C), 6, scale=C ** -0.5)
    W_o = _bf16((C, Hh * d), 7, scale=(Hh * d) ** -0.5)
    y = gla.gla_layer_forward(x.cuda(), W_in.cuda(), W_o.cuda(), 1, Hh, d, wl.T, wl.H, wl.W)
    torch.cuda.synchronize()
    assert gla.gla_get_device_status() == gla.GLA_OK
    ref = O.layer_forward(x.double().numpy().reshape(1, N, C), W_in.double().numpy(),
                          W_o.double().numpy(), Hh, d, wl.T, wl.H, wl.W, wl.rope_theta, wl.eps)
    err = rel_rms_bf16out(np64(y).reshape(1, N, C), ref["y"])
    print(f"layer 480p: y {rel_rms(np64(y).reshape(1, N, C), ref['y']):.3e} of the RMS, "
          f"{err:.3e} beyond bf16 rounding")
    assert err <= BF16_TOL
