"""The FMA-pipe exp2 of the softmax anchor kernel (an_ex2_poly2 in
csrc/anchor.cuh), emulated in fp32 with the constants read from the kernel
source: round-to-integer by adding 1.5 * 2^23, the degree-4 polynomial on the
remainder, the integer part added to the exponent field.  Checked against
2^x over the whole score range the kernel sees (|x| <= 16.35) and beyond."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "gated_bidirectional_linear_b200", "csrc", "anchor.cuh")


def _constants():
    src = open(SRC).read()
    body = src[src.index("void an_ex2_poly2("):]
    body = body[:body.index("\n}\n")]
    lits = []
    for m in re.finditer(r"(-?\d+\.\d*(?:e-?\d+)?)f", body):
        v = float(m.group(1))
        if v not in lits:
            lits.append(v)
    magic = [v for v in lits if abs(v) == 12582912.0]
    coef = [v for v in lits if 0.0 < v < 1.0]
    return magic[0], coef          # coef: c4, c3, c2, c1 in source order


def _ex2(x):
    magic, (c4, c3, c2, c1) = _constants()
    f32 = np.float32
    x = x.astype(np.float32)
    t = x + f32(magic)
    xr = t - f32(magic)
    f = x - xr
    p = ((((f32(c4) * f + f32(c3)) * f + f32(c2)) * f + f32(c1)) * f + f32(1.0))
    bits = p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23)
                                                   & 0xFFFFFFFF)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_magic_constant_has_nine_zero_low_bits():
    magic, coef = _constants()
    assert magic == 1.5 * 2 ** 23 and len(coef) == 4
    bits = int(np.float32(magic).view(np.uint32))
    assert bits & 0x1FF == 0


def test_relative_error_over_the_score_range():
    x = np.linspace(-16.4, 16.4, 2_000_001)
    got = _ex2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 4e-6, rel.max()


def test_integers_are_exact_and_wide_range():
    n = np.arange(-120, 121, dtype=np.float64)
    assert np.array_equal(_ex2(n).astype(np.float64), np.exp2(n))
    x = np.linspace(-100.0, 100.0, 200_001)
    rel = np.abs(_ex2(x).astype(np.float64) - np.exp2(x.astype(np.float32).astype(np.float64)))
    rel /= np.exp2(x.astype(np.float32).astype(np.float64))
    assert rel.max() < 4e-6
