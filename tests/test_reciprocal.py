"""The correction step of the quantize kernels' correctly rounded reciprocal,
checked exhaustively on the CPU.

The kernels need r = RN(1/a) for Markstein's quotient step (P. Markstein,
"Computation of elementary functions on the IBM RISC System/6000 processor",
IBM J. Res. Dev. 1990).  They take the hardware approximation, one Newton
step (which leaves a faithful y: one of the two floats around 1/a), then a
correction: e = 1 - a y in one FMA (exact), nb = the neighbour of y on the
side of 1/a, and the result is nb when |e| > a |nb - y| / 2, else y.

Here every fp32 significand of a in [1, 2) is run through that correction
from BOTH faithful starting points, with each FMA emulated as an exact
float64 product and difference followed by one rounding to float32.  The
result must equal RN(1/a) every time.  The step is scale-free over the range
the kernels use it in (a in [2^-96, 2^96]: 1/a normal, and a times half a gap
of y exact), so the significands cover every exponent.  The Newton step's
faithfulness rests on the hardware approximation's documented 1-ulp bound; the
GPU quantize tests (every fp32 v in [0, 1], thresholds' neighbourhoods over
the exponent range) check the whole path end to end.
"""
import numpy as np


def _rn32_reciprocal(a64):
    # RN32(1/a) via float64: 1/a is at least 2^-49 relative away from every
    # float32 midpoint (it is never one), far more than float64's 2^-53 error
    return (1.0 / a64).astype(np.float32)


def _correct(a, y):
    a64 = a.astype(np.float64)
    e64 = 1.0 - a64 * y.astype(np.float64)          # exact in float64
    e = e64.astype(np.float32)
    assert np.array_equal(e.astype(np.float64), e64), "1 - a y must be exact in fp32"
    yb = y.view(np.uint32)
    nb = np.where(e > 0, yb + np.uint32(1), yb - np.uint32(1)).view(np.float32)
    gap = np.abs(nb.astype(np.float64) - y.astype(np.float64))    # one ulp, exact
    half_gap = (a64 * (0.5 * gap)).astype(np.float32)
    assert np.array_equal(half_gap.astype(np.float64), a64 * 0.5 * gap)
    return np.where(np.abs(e) > half_gap, nb, y)


def test_correction_from_either_faithful_start_gives_rn_for_every_significand():
    a = (np.arange(1 << 23, dtype=np.uint32) | np.uint32(0x3F800000)).view(np.float32)
    a64 = a.astype(np.float64)
    want = _rn32_reciprocal(a64)
    inv = 1.0 / a64
    below = np.where(want.astype(np.float64) <= inv, want, np.nextafter(want, np.float32(0)))
    above = np.where(want.astype(np.float64) >= inv, want, np.nextafter(want, np.float32(np.inf)))
    for start in (below, above):
        got = _correct(a, start)
        bad = np.nonzero(got.view(np.uint32) != want.view(np.uint32))[0]
        assert bad.size == 0, (bad.size, a[bad[:4]])


def test_a_mistake_in_the_correction_is_caught():
    """Comparing against the full gap instead of half of it must fail."""
    a = (np.arange(1 << 16, dtype=np.uint32) * 128 | np.uint32(0x3F800000)).view(np.float32)
    a64 = a.astype(np.float64)
    want = _rn32_reciprocal(a64)
    inv = 1.0 / a64
    start = np.where(want.astype(np.float64) <= inv, want, np.nextafter(want, np.float32(0)))
    e = (1.0 - a64 * start.astype(np.float64)).astype(np.float32)
    nb = np.where(e > 0, start.view(np.uint32) + 1, start.view(np.uint32) - 1).view(np.float32)
    full_gap = (a64 * np.abs(nb.astype(np.float64) - start.astype(np.float64))).astype(np.float32)
    wrong = np.where(np.abs(e) > full_gap, nb, start)
    assert np.any(wrong.view(np.uint32) != want.view(np.uint32))
