"""libgla.so loads without a GPU, exports every entry point include/gla.h
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from gated_bidirectional_linear_b200 import gla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gla.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GLA_API\s+[\w\s\*]*?\b(gla_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for must in ("gla_forward", "gla_block_causal_step", "gla_forward_workspace_size",
                 "gla_forward_debug", "gla_get_device_status", "gla_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = gla.lib()
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    assert set(declared_symbols()) <= set(gla._SIGS)


def test_status_strings():
    assert gla.status_string(0) == "GLA_OK"
    for s in range(1, 6):
        assert gla.status_string(s).startswith("GLA_ERR_")
    assert gla.status_string(99) == "unknown gla_status"


def test_workspace_sizes():
    ws = gla.gla_forward_workspace_size(2, 20, 128, 16, 23, 40, gla.GLA_DTYPE_BF16)
    assert ws > (512 + 40) * 128 * 128 * 4
    assert gla.gla_forward_workspace_size(1, 2, 48, 2, 4, 4, 0) == 0      # bad head dim
    assert gla.gla_forward_workspace_size(0, 2, 32, 2, 4, 4, 0) == 0      # bad batch
    assert gla.gla_block_causal_workspace_size(1, 20, 128, 3, 23, 40, 1) < ws
    arena = gla.gla_forward_host_arena_size(1, 2, 32, 2, 4, 4, 0)
    assert arena >= 6 * 32 * 2 * 32 * 4


FAKE = 1 << 20          # a 16-byte aligned address that is never dereferenced


def _fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=FAKE, g=FAKE, B=1, Hh=2, d=32, T=2, H=4, W=4,
             theta=1e4, eps=1e-6, dtype=0, out=FAKE, ws=FAKE, wsb=1 << 30, stream=None,
             path=0)
    a.update(kw)
    return gla.lib().gla_forward_ex(a["q"], a["k"], a["v"], a["beta"], a["g"], a["B"], a["Hh"],
                                    a["d"], a["T"], a["H"], a["W"], a["theta"], a["eps"],
                                    a["dtype"], a["out"], a["ws"], a["wsb"], a["stream"],
                                    a["path"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), gla.GLA_ERR_INVALID_ARG),
    (dict(out=None), gla.GLA_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), gla.GLA_ERR_INVALID_ARG),          # misaligned
    (dict(d=48), gla.GLA_ERR_INVALID_ARG),
    (dict(T=0), gla.GLA_ERR_INVALID_ARG),
    (dict(eps=0.0), gla.GLA_ERR_INVALID_ARG),
    (dict(eps=float("nan")), gla.GLA_ERR_INVALID_ARG),
    (dict(dtype=7), gla.GLA_ERR_INVALID_ARG),
    (dict(path=gla.GLA_PATH_TENSOR), gla.GLA_ERR_UNSUPPORTED),   # fp32 has no tensor path
    (dict(path=9), gla.GLA_ERR_UNSUPPORTED),
    (dict(ws=None), gla.GLA_ERR_WORKSPACE),
    (dict(ws=FAKE + 16), gla.GLA_ERR_WORKSPACE),           # not 256-byte aligned
    (dict(wsb=1024), gla.GLA_ERR_WORKSPACE),
])
def test_forward_rejects_bad_arguments(kw, status):
    assert _fwd(**kw) == status


def test_block_step_rejects_bad_arguments():
    lib = gla.lib()
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 32, 2, 4, 4, 0, 1e4, 1e-6, 0,
            FAKE, FAKE, 1 << 30, None, 0]
    bad_state = list(args); bad_state[0] = None
    assert lib.gla_block_causal_step_ex(*bad_state) == gla.GLA_ERR_INVALID_ARG
    bad_t0 = list(args); bad_t0[13] = -1
    assert lib.gla_block_causal_step_ex(*bad_t0) == gla.GLA_ERR_INVALID_ARG
    small = list(args); small[19] = 64
    assert lib.gla_block_causal_step_ex(*small) == gla.GLA_ERR_WORKSPACE


def test_host_entry_rejects_bad_arguments():
    lib = gla.lib()
    args = [FAKE] * 5 + [1, 2, 32, 2, 4, 4, 1e4, 1e-6, 0, FAKE, FAKE, 1 << 30, None]
    no_out = list(args); no_out[14] = None
    assert lib.gla_forward_host(*no_out) == gla.GLA_ERR_INVALID_ARG
    small = list(args); small[16] = 1024
    assert lib.gla_forward_host(*small) == gla.GLA_ERR_WORKSPACE


def test_plan_paths():
    # tensor path: the state reduction walks 96-token tiles
    assert gla.gla_plan(2, 20, 128, 16, 23, 40, 1, 0, 148) == (148, 96, gla.GLA_PATH_TENSOR)
    assert gla.gla_plan(1, 2, 32, 2, 4, 4, 0, 0, 148) == (2, 64, gla.GLA_PATH_SIMT)
    assert gla.gla_plan(2, 20, 128, 16, 23, 40, 1, gla.GLA_PATH_SIMT, 148)[2] == gla.GLA_PATH_SIMT
    # 20 heads x 29 tiles of 96 tokens = 580 items >= 148 CTAs
    assert gla.gla_plan(1, 20, 128, 3, 23, 40, 1, 0, 148)[0] == 148
    # fewer items than SMs: one CTA per item (2 heads x 2 tiles of 96 tokens)
    assert gla.gla_plan(1, 2, 128, 1, 1, 100, 1, 0, 148)[0] == 4
    with pytest.raises(gla.GlaError):
        gla.gla_plan(1, 2, 32, 2, 4, 4, 0, gla.GLA_PATH_TENSOR, 148)


def test_selftest_rejects_out_of_range_limits():
    # Rejected before anything is launched, so no GPU is needed.
    lib = gla.lib()
    assert lib.gla_selftest_wait_timeout(0, None) == gla.GLA_ERR_INVALID_ARG
    assert lib.gla_selftest_wait_timeout(1000001, None) == gla.GLA_ERR_INVALID_ARG
