"""Exact-arithmetic restatement of 4-bit blockwise quantization, for tiny inputs.

TEST INFRASTRUCTURE ONLY.  It pins the C oracle: every quantity is a
``fractions.Fraction``.  Rounding to a binary format is written out from the
IEEE 754 definition (round to nearest, ties to even).  Nothing here is shared
with ``bnb4_oracle.c``: the code tables are rebuilt from their own
definitions, and the fp32 quotient is the exact quotient rounded once.
"""
from __future__ import annotations

import struct
from fractions import Fraction

# The NF4 decimal literals of the 4096x4096 gemv workload, as text.
NF4_LITERALS = [
    "-1", "-0.6961928", "-0.5250731", "-0.3949175", "-0.2844414", "-0.1848074",
    "-0.0910500", "0", "0.0795803", "0.1609302", "0.2461123", "0.3379152",
    "0.4407098", "0.5626170", "0.7229568", "1",
]

# (significand bits incl. the implicit one, minimum normal exponent, maximum exponent)
FORMATS = {"f32": (24, -126, 127), "f16": (11, -14, 15), "bf16": (8, -126, 127)}


def round_to(q: Fraction, fmt: str):
    """Round an exact rational to the nearest value of a binary format, ties to even.

    Returns a Fraction, or float('inf') / float('-inf') on overflow.
    """
    p, emin, emax = FORMATS[fmt]
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    # exponent of the leading bit: 2**e <= a < 2**(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - (p - 1))
    r = round(a / quantum) * quantum  # Python's round() of a Fraction is half-to-even
    maxf = (2 - Fraction(2) ** (1 - p)) * Fraction(2) ** emax
    if r > maxf:
        return float("inf") * sign
    return sign * r


def exact(v) -> Fraction:
    return Fraction(float(v))


def f16_bits_to_fraction(h: int) -> Fraction:
    s, e, m = (h >> 15) & 1, (h >> 10) & 31, h & 1023
    assert e != 31, "inf/nan not used"
    v = Fraction(m, 1 << 24) if e == 0 else Fraction(1024 + m) * Fraction(2) ** (e - 25)
    return -v if s else v


def bf16_bits_to_fraction(h: int) -> Fraction:
    s, e, m = (h >> 15) & 1, (h >> 7) & 255, h & 127
    assert e != 255, "inf/nan not used"
    v = Fraction(m) * Fraction(2) ** (-133) if e == 0 else Fraction(128 + m) * Fraction(2) ** (e - 134)
    return -v if s else v


def f32_bits_to_fraction(b: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", b))[0])


def nf4_table() -> list:
    return [round_to(Fraction(s), "f32") for s in NF4_LITERALS]


def fp4_table() -> list:
    """E2M1, bias 1, subnormals; magnitude / 6; index = s<<3 | e<<1 | m."""
    out = []
    for idx in range(16):
        s, e, m = (idx >> 3) & 1, (idx >> 1) & 3, idx & 1
        mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
        v = round_to(mag / 6, "f32")
        out.append(-v if s else v)
    return out


def table(qtype: str) -> list:
    return nf4_table() if qtype == "nf4" else fp4_table()


def quantize(values: list, blocksize: int, qtype: str):
    """values: exact Fractions (already representable in the input dtype).

    Returns (packed bytes list, absmax list of Fractions, code indices list).
    """
    codes = table(qtype)
    n = len(values)
    idxs, absmax = [], []
    for lo in range(0, n, blocksize):
        blk = values[lo:lo + blocksize]
        a = max(abs(v) for v in blk)
        absmax.append(a)
        for x in blk:
            v = Fraction(0) if a == 0 else round_to(x / a, "f32")
            dists = [abs(v - c) for c in codes]
            best = min(range(16), key=lambda i: (dists[i], i))
            idxs.append(best)
    packed = []
    for j in range(0, n, 2):
        hi = idxs[j]
        lo_ = idxs[j + 1] if j + 1 < n else 0
        packed.append((hi << 4) | lo_)
    return packed, absmax, idxs


def dequantize(idxs: list, absmax: list, blocksize: int, qtype: str, out_fmt: str) -> list:
    codes = table(qtype)
    out = []
    for i, q in enumerate(idxs):
        p = round_to(codes[q] * absmax[i // blocksize], "f32")
        out.append(p if out_fmt == "f32" else round_to(p, out_fmt))
    return out


def matmul(X: list, W: list, bias=None) -> list:
    """Exact Y = X @ W^T (+ bias): X [M][K], W [N][K] of Fractions."""
    Y = []
    for row in X:
        Y.append([sum((a * b for a, b in zip(row, wr)), Fraction(0)) + (bias[j] if bias else 0)
                  for j, wr in enumerate(W)])
    return Y


def quantize_with_table(values: list, blocksize: int, codes: list):
    """Blockwise quantization against any ascending table of exact Fractions:
    (code indices, absmax list), one index per element, ties to the smallest index."""
    idxs, absmax = [], []
    for lo in range(0, len(values), blocksize):
        blk = values[lo:lo + blocksize]
        a = max(abs(v) for v in blk)
        absmax.append(a)
        for x in blk:
            v = Fraction(0) if a == 0 else round_to(x / a, "f32")
            best = min(range(len(codes)), key=lambda i: (abs(v - codes[i]), i))
            idxs.append(best)
    return idxs, absmax


def dequantize_with_table(idxs: list, absmax: list, blocksize: int, codes: list, out_fmt: str) -> list:
    out = []
    for i, q in enumerate(idxs):
        p = round_to(codes[q] * absmax[i // blocksize], "f32")
        out.append(p if out_fmt == "f32" else round_to(p, out_fmt))
    return out
