"""Inputs that sit on the knife edges of 4-bit quantization, found by exact search.

* ``division_blocks``: blocks [a, x] whose element x lies within a few fp32
  ulps of a decision threshold (the midpoint between two neighbouring codes),
  chosen so that the IEEE quotient x / a and the cheaper x * fp32(1 / a) pick
  different codes.  Any implementation that normalises with a reciprocal
  instead of the true quotient fails on them.
* ``double_rounding_pairs``: (code index, absmax) pairs whose fp32 product,
  rounded once more to bf16 / fp16, differs from rounding the exact product
  straight to that dtype.  They pin "one fp32 product, then one conversion".

Everything is computed with ``fractions.Fraction`` and the exact rounding of
``oracle.bruteforce``; no value comes from the code under test.
"""
from __future__ import annotations

import random
from fractions import Fraction

import numpy as np

from oracle import bruteforce as bf


def _ulp32(v: Fraction) -> Fraction:
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    return Fraction(2) ** (max(e, -126) - 23)


def _nearest(v: Fraction, codes) -> int:
    d = [abs(v - c) for c in codes]
    return min(range(16), key=lambda i: (d[i], i))


def division_blocks(qtype: str, blocksize: int, seed: int = 0, per_threshold: int = 2):
    """Returns a float32 array of whole blocks; each block is [a, x, 0, ..., 0]."""
    rnd = random.Random(seed * 7919 + (0 if qtype == "nf4" else 1))
    codes = bf.table(qtype)
    vals = sorted(set(codes))
    mids = [(p + q) / 2 for p, q in zip(vals, vals[1:])]
    blocks = []
    for m in mids:
        found = 0
        for _ in range(4000):
            if found >= per_threshold:
                break
            a = bf.round_to(Fraction(rnd.uniform(0.25, 64.0)), "f32")
            x0 = bf.round_to(m * a, "f32")
            u = _ulp32(x0)
            for k in range(-3, 4):
                x = x0 + k * u
                if abs(x) > a:
                    continue
                v_div = bf.round_to(x / a, "f32")
                v_rcp = bf.round_to(x * bf.round_to(1 / a, "f32"), "f32")
                if _nearest(v_div, codes) != _nearest(v_rcp, codes):
                    blocks.append((a, x))
                    found += 1
                    break
    out = np.zeros(len(blocks) * blocksize, np.float32)
    for i, (a, x) in enumerate(blocks):
        out[i * blocksize] = float(a)
        out[i * blocksize + 1] = float(x)
    return out


def _round_dtype_np(d: np.ndarray, mant_bits: int, emin: int) -> np.ndarray:
    """Round float64 values (exact, <= 48 significant bits) to p = mant_bits+1 bits."""
    a = np.abs(d)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # guard the floor(log2) against values just below a power of two
    e = np.where(2.0 ** e > a, e - 1, e)
    e = np.where(2.0 ** (e + 1) <= a, e + 1, e)
    e = np.maximum(e, emin)
    q = 2.0 ** (e - mant_bits)
    return np.sign(d) * np.rint(a / q) * q


def double_rounding_pairs(qtype: str, out_dtype: str, want: int = 8, seed: int = 0):
    """(code index, absmax) pairs where RN_dt(RN32(c*a)) != RN_dt(c*a)."""
    mant, emin = {"bf16": (7, -126), "f16": (10, -14)}[out_dtype]
    codes = np.array([float(c) for c in bf.table(qtype)], np.float64)
    rng = np.random.default_rng(seed)
    pairs = []
    lo = 0.5 if out_dtype == "bf16" else 0.01
    hi = 1000.0 if out_dtype == "bf16" else 60000.0
    for _ in range(64):
        a = rng.uniform(lo, hi, size=200_000).astype(np.float32)
        for ci in range(16):
            if codes[ci] == 0.0 or abs(codes[ci]) == 1.0:
                continue
            exact = codes[ci] * a.astype(np.float64)           # exact: 24 x 24 bits
            via32 = exact.astype(np.float32).astype(np.float64)  # RN to fp32
            r1 = _round_dtype_np(via32, mant, emin)
            r2 = _round_dtype_np(exact, mant, emin)
            hit = np.nonzero(r1 != r2)[0]
            for h in hit[:2]:
                pairs.append((ci, float(a[h])))
            if len(pairs) >= want:
                return pairs
    return pairs


def threshold_neighbourhoods(qtype: str, blocksize: int = 64, n_scales: int = 2048,
                             radius: int = 4, seed: int = 0):
    """Blocks [a, x, x, ...] where every x lies within `radius` fp32 steps of a
    decision threshold scaled by a, for n_scales absmax values a spread over
    the whole exponent range.  Returns a float32 array of whole blocks."""
    rng = np.random.default_rng(seed)
    vals = sorted(set(float(c) for c in bf.table(qtype)))
    mids = np.array([(p + q) / 2 for p, q in zip(vals, vals[1:])], np.float64)  # exact
    exps = rng.integers(-126, 128, size=n_scales)
    exps[:8] = [-126, -97, -96, -95, 95, 96, 97, 127]
    mant = rng.uniform(1.0, 2.0, size=n_scales)
    a = (mant * np.exp2(exps.astype(np.float64))).astype(np.float32)
    a = a[np.isfinite(a) & (a > 0)]
    xs = []
    for ai in a:
        x0 = (mids * np.float64(ai)).astype(np.float32)   # exact product, one rounding
        cand = [x0]
        up, dn = x0.copy(), x0.copy()
        for _ in range(radius):
            up = np.nextafter(up, np.float32(np.inf))
            dn = np.nextafter(dn, np.float32(-np.inf))
            cand += [up, dn]
        c = np.concatenate(cand)
        c = c[np.abs(c) <= ai]
        xs.append((ai, c))
    per = blocksize - 1
    blocks = []
    for ai, c in xs:
        for j in range(0, c.size, per):
            blk = np.zeros(blocksize, np.float32)
            blk[0] = ai
            part = c[j:j + per]
            blk[1:1 + part.size] = part
            blocks.append(blk)
    return np.concatenate(blocks)
