"""Why NF4 with bf16 inputs needs no exact redo in the quantize kernel.

The kernel's screen compares x * RN(1/a) with a key per NF4 threshold.  With
bf16 inputs every ratio x / a (|x| <= a, both with 8-bit significands) lies
at least two ulps -- in fact 15 -- from every NF4 midpoint, so the IEEE
quotient falls on the same side of the threshold as the ratio, and a key put
in the gap between the nearest ratios decides every element exactly.  fp16
ratios (11-bit significands) come within a fraction of an ulp of some
midpoints, so fp16 keeps the redo.  Checked by enumerating every ratio of
significands at every scaling that reaches a midpoint.
"""
import math

import numpy as np
import pytest

from oracle import bruteforce as bf


def nf4_midpoint_magnitudes():
    c = [float(v) for v in bf.nf4_table()]          # the fp32 NF4 codes, exactly
    return sorted({abs((a + b) / 2) for a, b in zip(c, c[1:])})


def nearest_ratio_ulps(p):
    A = np.arange(1 << (p - 1), 1 << p, dtype=np.float64)
    X = np.arange(0, 1 << p, dtype=np.float64)
    R = np.unique((X[None, :] / A[:, None]).ravel())   # ratio significands
    out = []
    for m in nf4_midpoint_magnitudes():
        best = math.inf
        for d in range(-14, 2):
            v = R * 2.0 ** d
            i = int(np.searchsorted(v, m))
            for j in (i - 1, i):
                if 0 <= j < v.size:
                    best = min(best, abs(v[j] - m))
        out.append(best / 2.0 ** (math.floor(math.log2(m)) - 23))
    return out


def test_bf16_ratios_stay_clear_of_nf4_midpoints():
    ulps = nearest_ratio_ulps(8)
    assert len(ulps) == 15
    assert min(ulps) >= 2, min(ulps)      # the table builder's condition
    assert min(ulps) > 15, min(ulps)      # the margin measured for NF4


def test_fp16_ratios_come_near_nf4_midpoints():
    assert min(nearest_ratio_ulps(11)) < 2
