"""The gap that lets the FP4 screen decide 16-bit inputs exactly.

FP4 codes are E2M1 values / 6, so the decision points are T = k / 24.  The
quantize kernel's FP4 keys for bf16 and fp16 inputs rest on this fact: a ratio
x / a of two values with p-bit significands (x <= a) either equals T or lies
at least g_T = 2^(e_T - p) / 24 from it, e_T the smallest integer above
log2 T - 1.  Checked here by brute force over every pair of significands and
every exponent difference that can bring x / a near T.
"""
import math

import numpy as np
import pytest

DECISION_POINTS = (1, 3, 5, 7, 10, 14, 20)   # k of T = k / 24: midpoints of E2M1 / 6 magnitudes


def gap_bound(k: int, p: int) -> float:
    T = k / 24
    e = math.floor(math.log2(T) - 1.0 - 1e-9) + 1
    return 2.0 ** (e - p) / 24


def test_decision_points_are_the_e2m1_midpoints():
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]            # E2M1 magnitudes
    mids = [(a + b) / 2 / 6 for a, b in zip(mags, mags[1:])]
    assert [round(m * 24, 9) for m in mids] == list(DECISION_POINTS)


@pytest.mark.parametrize("p", [8, 11])   # bf16, fp16 significand bits
def test_ratios_of_16bit_values_keep_clear_of_fp4_decision_points(p):
    A = np.arange(1 << (p - 1), 1 << p, dtype=np.int64)[:, None]   # normal a
    X = np.arange(0, 1 << p, dtype=np.int64)[None, :]               # any x, subnormal included
    for k in DECISION_POINTS:
        best = np.inf
        hits = 0
        for d in range(-12, 1):                # ex - ea; x / a < 2^(d + 1)
            s = 1 << (-d)
            num = np.abs(24 * X - k * A * s)   # |24 x - k a| / 2^ex
            hits += int((num == 0).sum())
            dist = num[num != 0] / (24 * np.broadcast_to(A, num.shape)[num != 0] * s)
            best = min(best, float(dist.min()))
        assert hits > 0, "x / a lands exactly on T for some pairs"
        assert best >= gap_bound(k, p), (k, best, gap_bound(k, p))
        # the key sits half a gap out, moved by at most 8 ulps (<= 8 T 2^-23)
        # for its rank nibble: still further than the screen's error (T 2^-24)
        # from both T and T +- g_T
        T = k / 24
        assert gap_bound(k, p) / 2 - 8 * T * 2.0 ** -23 > T * 2.0 ** -24
