"""The read-out's RoPE table copies, checked on the host (no GPU).

Each read-out CTA brings its window of the RoPE table into shared memory by
bulk copies from the whole-call table.  A bulk copy needs 16-byte aligned
addresses and sizes, so a plan that broke that would fault the GPU; one that
mapped a row wrongly would rotate tokens by the wrong angles.  The library's
own plan code is run here through gla_check_rope_copy for the benchmarked
shapes, their neighbours and random grids."""
import random

import pytest

from gated_bidirectional_linear_b200 import gla, workloads

SMS = (148, 132, 37, 5, 1)


@pytest.mark.parametrize("name", ["480p", "720p", "14b", "blk"])
@pytest.mark.parametrize("sms", SMS)
def test_workload_shapes(name, sms):
    wl = workloads.WORKLOADS[name]
    assert gla.gla_check_rope_copy(wl.batch, wl.heads, 128, wl.T, wl.H, wl.W, sms) == gla.GLA_OK


@pytest.mark.parametrize("seed", range(60))
def test_random_grids(seed):
    rnd = random.Random(seed)
    B, Hh = rnd.randint(1, 3), rnd.randint(1, 40)
    T, H, W = rnd.randint(1, 70), rnd.randint(1, 48), rnd.randint(1, 48)
    sms = rnd.choice(SMS)
    assert gla.gla_check_rope_copy(B, Hh, 128, T, H, W, sms) == gla.GLA_OK


def test_rejects_what_the_tensor_path_does_not_take():
    assert gla.gla_check_rope_copy(1, 2, 32, 2, 4, 4, 148) == gla.GLA_ERR_UNSUPPORTED
    assert gla.gla_check_rope_copy(0, 2, 128, 2, 4, 4, 148) == gla.GLA_ERR_INVALID_ARG
