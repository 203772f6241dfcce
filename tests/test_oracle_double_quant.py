"""Pins for the oracle's double quantization of absmax (reading R9).

"mps-bitsandbytes 0.4.7", Functional API, Double Quantization: the pages give
double_quant(absmax, double_quant_block=256) -> (absmax_quant, absmax_scales)
and dequant_absmax, not the arithmetic.  The checks below fix the reading
with an exact rational restatement (every fp32 rounding done on Fractions),
closed forms and special cases, so that a plausible slip in the C code (a
truncation instead of a rounding, the wrong maximum, another rounding order)
fails one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import bruteforce as bf


def _exact_double_quant(a, group):
    """R9 on exact rationals: each fp32 operation is rounded once by round_to."""
    n = len(a)
    q, scales = [], []
    for g0 in range(0, n, group):
        blk = a[g0:g0 + group]
        s = Fraction(0)
        for v in blk:
            if not math.isnan(v) and Fraction(v) > s:
                s = Fraction(v)
        scales.append(s)
        for v in blk:
            code = 0
            if s > 0 and not math.isnan(v):
                quo = bf.round_to(Fraction(v) / s, "f32")
                t = bf.round_to(quo * 255, "f32")
                r = round(t)  # half to even
                if r > 0:
                    code = min(r, 255)
            q.append(code)
    return q, scales


def _exact_dequant(q, scales, group):
    out = []
    for i, c in enumerate(q):
        step = bf.round_to(scales[i // group] / 255, "f32")
        out.append(bf.round_to(c * step, "f32"))
    return out


@pytest.mark.parametrize("group", [4, 7, 256])
def test_double_quant_matches_exact_rationals(group):
    rng = np.random.default_rng(group)
    # absmax-like values over several binades, a few exact ties of the 255-step grid
    a = (rng.lognormal(-3.0, 1.5, 3 * group + 5)).astype(np.float32)
    a[::11] = np.float32(0.0)
    a[3] = a[:group].max() * np.float32(0.5)          # v = 1/2 -> 127.5: ties to even
    q, s = oracle.double_quant(a, group)
    qe, se = _exact_double_quant([float(v) for v in a], group)
    assert list(q) == qe
    assert [Fraction(float(v)) for v in s] == se
    out = oracle.dequant_absmax(q, s, group)
    oute = _exact_dequant(qe, se, group)
    assert [Fraction(float(v)) for v in out] == oute


def test_double_quant_closed_forms():
    # scale 255: integer absmax k quantizes to k and comes back exactly
    a = np.arange(256, dtype=np.float32)
    a[255] = 255.0
    q, s = oracle.double_quant(a, 256)
    assert s[0] == 255.0
    assert np.array_equal(q, np.arange(256, dtype=np.uint8))
    assert np.array_equal(oracle.dequant_absmax(q, s, 256), a)
    # the group maximum is code 255; a half-scale value is the tie 127.5 -> 128
    q, s = oracle.double_quant(np.array([3.0, 1.5, 6.0], np.float32), 3)
    assert s[0] == 6.0 and list(q) == [128, 64, 255]   # 0.5*255 = 127.5 -> 128, 63.75 -> 64


def test_double_quant_special_values():
    nan = np.float32("nan")
    a = np.array([0.0, -0.0, 0.0, 0.0,   nan, 2.0, -1.0, 1.0], np.float32)
    q, s = oracle.double_quant(a, 4)
    assert s[0] == 0.0 and not math.copysign(1.0, float(s[0])) < 0   # +0 for an all-zero group
    assert list(q[:4]) == [0, 0, 0, 0]
    assert s[1] == 2.0                      # NaN skipped by the maximum
    assert list(q[4:]) == [0, 255, 0, 128]  # NaN -> 0, negative -> 0, 1/2 -> 127.5 -> 128
    assert np.all(oracle.dequant_absmax(q[:4], s[:1], 4) == 0.0)


def test_double_quant_error_bound_and_ragged_tail():
    rng = np.random.default_rng(7)
    a = rng.lognormal(-4.0, 2.0, 1000).astype(np.float32)   # 1000 = 3 groups of 256 + 232
    q, s = oracle.double_quant(a, 256)
    assert s.size == 4
    for g in range(4):
        assert s[g] == a[256 * g:256 * (g + 1)].max()
    out = oracle.dequant_absmax(q, s, 256).astype(np.float64)
    scale = np.repeat(s.astype(np.float64), 256)[:1000]
    # half a step of scale/255, plus the two fp32 roundings
    assert np.all(np.abs(out - a) <= scale / 510 * (1 + 2.0 ** -20) + scale * 2.0 ** -23)
