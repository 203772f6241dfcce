"""Pins for the oracle's 8-bit blockwise quantization (reading R10), CPU only.

"Feat/mps gemm 4bit bf16", What runs natively now (quantize_blockwise /
dequantize_blockwise) and Correctness (the int8 kernel checked against an
exact float64 reference; an oracle that snapped the normalised value to a
65536-point grid missed 1365 of 1,048,576 values).  The pages print no 8-bit
code table, so the table is an argument.  Each pin checks the oracle against
something other than itself:
  * the exact rational restatement (oracle.bruteforce) on tiny inputs;
  * a closed form for a dyadic linear table;
  * exact comparisons at every midpoint's fp32 neighbours (what a grid snap
    gets wrong);
  * special blocks, idempotence and the error bound;
  * double rounding in the dequantization.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import bruteforce as bf
import synthetic


def _to_fracs(arr, dtype):
    if dtype == "f32":
        return [Fraction(float(v)) for v in arr]
    conv = bf.f16_bits_to_fraction if dtype == "f16" else bf.bf16_bits_to_fraction
    return [conv(int(v)) for v in arr]


def _table(kind: str, seed: int = 0) -> np.ndarray:
    """256 strictly ascending fp32 entries in [-1, 1], each 0 or >= 2^-24 in magnitude.
    uniform: spread evenly; log: magnitudes log-uniform down to 2^-24 (a dynamic
    range like an exponent-coded table); both hold -1, 0 and 1."""
    rng = np.random.default_rng(seed)
    vals = {-1.0, 0.0, 1.0}
    while len(vals) < 256:
        if kind == "uniform":
            v = float(np.float32(rng.uniform(-1.0, 1.0)))
        else:
            v = float(np.float32(rng.choice([-1.0, 1.0]) * 2.0 ** rng.uniform(-24.0, 0.0)))
        if v == 0.0 or abs(v) >= 2.0 ** -24:
            vals.add(v)
    return np.array(sorted(vals), np.float32)


def _dyadic() -> np.ndarray:
    return ((np.arange(256) - 128) / 128.0).astype(np.float32)   # -1 .. 127/128, exact


# ------------------------------------------------------------ exact rationals

@pytest.mark.parametrize("kind", ["uniform", "log"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("n,B", [(1, 4), (5, 4), (64, 64), (65, 64), (130, 64), (37, 8)])
def test_matches_exact_rationals(kind, dtype, n, B):
    code = _table(kind, seed=n + B)
    x = synthetic.storage_numpy(synthetic.normal((n,), n * 7 + B, 1.0, dtype,
                                                 outlier_frac=0.05)).reshape(-1)
    q, a = oracle.quantize_8bit(x, dtype, B, code)
    codes = [Fraction(float(c)) for c in code]
    idxs, amax = bf.quantize_with_table(_to_fracs(x, dtype), B, codes)
    assert list(q) == idxs
    assert [Fraction(float(v)) for v in a] == amax
    for out in ("f32", "f16", "bf16"):
        got = oracle.dequantize_8bit(q, a, n, B, code, out)
        want = bf.dequantize_with_table(idxs, amax, B, codes, out)
        assert _to_fracs(got, out) == want, out


# -------------------------------------------------------------- closed form

def test_dyadic_linear_table_closed_form():
    """code_j = (j - 128)/128: the nearest index of v is 128 v + 128 rounded
    half down (ties to the smaller index), clamped to [0, 255].  Blocks start
    with 1.0, so absmax is 1 and v = x exactly."""
    rng = np.random.default_rng(3)
    v = rng.uniform(-1.0, 1.0, 200_000).astype(np.float32)
    ties = ((np.arange(-128, 128) + 0.5) / 128.0).astype(np.float32)        # exact midpoints
    near = np.concatenate([np.nextafter(ties, np.float32(-2)), np.nextafter(ties, np.float32(2))])
    v = np.concatenate([v, ties, near, np.float32([-1.0, 0.0, 1.0, 127 / 128, 0.99999994])])
    v = v[np.abs(v) <= 1.0]
    B = 64
    nb = -(-v.size // (B - 1))
    x = np.zeros(nb * B, np.float32)
    x[0::B] = 1.0
    mask = np.ones(nb * B, bool)
    mask[0::B] = False
    x[np.nonzero(mask)[0][:v.size]] = v
    q, a = oracle.quantize_8bit(x, "f32", B, _dyadic())
    assert np.all(a == 1.0)
    t = 128.0 * x.astype(np.float64) + 128.0                                 # exact
    want = np.clip(np.ceil(t - 0.5), 0, 255).astype(np.uint8)
    assert np.array_equal(q, want)


# -------------------------------------------------- midpoint neighbourhoods

@pytest.mark.parametrize("kind", ["uniform", "log"])
def test_every_midpoint_neighbourhood(kind):
    """For every pair of adjacent entries, the fp32 values nearest their exact
    midpoint and two steps around it, decided by exact rational comparison.
    A search that snaps v to a 65536-point grid first fails here."""
    code = _table(kind, seed=11)
    codes = [Fraction(float(c)) for c in code]
    vs, want = [], []
    for j in range(255):
        m = (codes[j] + codes[j + 1]) / 2
        m32 = np.float32(float(m))
        cands = [m32]
        for _ in range(2):
            cands.append(np.nextafter(cands[-1], np.float32(2)))
        c = m32
        for _ in range(2):
            c = np.nextafter(c, np.float32(-2))
            cands.append(c)
        for v in cands:
            if not (code[j] <= v <= code[j + 1]):
                continue
            fv = Fraction(float(v))
            vs.append(v)
            want.append(j if abs(fv - codes[j]) <= abs(fv - codes[j + 1]) else j + 1)
    B = 64
    vs = np.array(vs, np.float32)
    nb = -(-vs.size // (B - 1))
    x = np.zeros(nb * B, np.float32)
    x[0::B] = 1.0
    pos = np.nonzero(np.arange(nb * B) % B != 0)[0][:vs.size]
    x[pos] = vs
    q, _ = oracle.quantize_8bit(x, "f32", B, code)
    bad = np.nonzero(q[pos] != np.array(want, np.uint8))[0]
    assert bad.size == 0, (bad.size, vs[bad[:4]])


# ------------------------------------------------ special blocks and bounds

def test_special_blocks():
    code = _table("uniform", seed=2)
    i0, im, ip = int(np.nonzero(code == 0)[0][0]), 0, 255
    x = np.array([0.0, 0.0, -0.0, 0.0,          # all-zero block: absmax 0, index of code 0
                  3.0, -3.0, 1.5, 0.0,          # +-absmax map to +-1
                  -0.0, 2.0, 0.0, 0.0], np.float32)
    q, a = oracle.quantize_8bit(x, "f32", 4, code)
    assert list(a) == [0.0, 3.0, 2.0]
    assert list(q[:4]) == [i0] * 4
    assert q[4] == ip and q[5] == im and q[7] == i0
    assert q[8] == i0 and q[9] == ip
    d = oracle.dequantize_8bit(q, a, x.size, 4, code, "f32")
    assert d[4] == 3.0 and d[5] == -3.0 and d[9] == 2.0 and np.all(d[:4] == 0.0)


@pytest.mark.parametrize("table", ["dyadic", "uniform_gapped"])
def test_error_bound_and_idempotence(table):
    if table == "dyadic":
        code = np.concatenate([_dyadic()[1:], np.float32([1.0])])   # -127/128 .. 127/128, 1
        code[0] = -1.0
    else:  # uniform with a minimum gap of 2^-12, so that re-quantization is stable
        rng = np.random.default_rng(5)
        g = rng.uniform(1.0, 3.0, 255)
        c = np.concatenate([[0.0], np.cumsum(g)]) / np.sum(g) * 2.0 - 1.0
        code = np.unique(np.float32(c))
        assert code.size == 256 and np.diff(code.astype(np.float64)).min() > 2.0 ** -12
        code[0], code[-1] = -1.0, 1.0
    assert np.all(np.diff(code) > 0)
    B = 64
    x = synthetic.normal((B * 40,), 8, 1.0, "f32", outlier_frac=0.02).numpy()
    q, a = oracle.quantize_8bit(x, "f32", B, code)
    d = oracle.dequantize_8bit(q, a, x.size, B, code, "f32").astype(np.float64)
    c64 = code.astype(np.float64)
    amax = np.repeat(a.astype(np.float64), B)
    v = x / amax
    # half the gap between the two entries around v, scaled, plus the fp32 roundings
    hi = np.clip(np.searchsorted(c64, v), 1, 255)
    gap = c64[hi] - c64[hi - 1]
    assert np.all(np.abs(d - x) <= amax * (gap / 2 + 2.0 ** -23) + np.abs(d) * 2.0 ** -24)
    q2, a2 = oracle.quantize_8bit(d.astype(np.float32), "f32", B, code)
    assert np.array_equal(a2, a) and np.array_equal(q2, q)


def _round_np(d: np.ndarray, mant_bits: int, emin: int) -> np.ndarray:
    """Round exact float64 values (<= 48 significant bits) to mant_bits+1 bits, ties to even."""
    a = np.abs(d)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(2.0 ** e > a, e - 1, e)
    e = np.where(2.0 ** (e + 1) <= a, e + 1, e)
    q = 2.0 ** (np.maximum(e, emin) - mant_bits)
    return np.sign(d) * np.rint(a / q) * q


def test_dequant_double_rounding():
    """(entry, absmax) pairs where rounding code*absmax straight to bf16 / fp16
    differs from rounding it to fp32 first: the oracle must round twice.  The
    search runs on exact float64 products (24 x 24 bits); the pairs found are
    then checked with exact rationals."""
    code = _table("uniform", seed=9)
    rng = np.random.default_rng(1)
    for out, mant, emin, lo, hi in (("bf16", 7, -126, 0.5, 1000.0), ("f16", 10, -14, 0.01, 60000.0)):
        found = []
        a = rng.uniform(lo, hi, 100_000).astype(np.float32)
        for j in rng.permutation(np.arange(1, 255))[:40]:
            exact = float(code[j]) * a.astype(np.float64)
            via32 = exact.astype(np.float32).astype(np.float64)
            hit = np.nonzero(_round_np(exact, mant, emin) != _round_np(via32, mant, emin))[0]
            found += [(int(j), a[h]) for h in hit[:1]]
            if len(found) >= 4:
                break
        assert len(found) >= 4, out
        for j, aa in found:   # the search's claim, checked exactly
            ex = Fraction(float(code[j])) * Fraction(float(aa))
            assert bf.round_to(ex, out) != bf.round_to(bf.round_to(ex, "f32"), out)
        q = np.array([j for j, _ in found], np.uint8)
        amax = np.array([aa for _, aa in found], np.float32)
        got = oracle.dequantize_8bit(q, amax, q.size, 1, code, out)
        want = [bf.round_to(bf.round_to(Fraction(float(code[j])) * Fraction(float(aa)), "f32"), out)
                for j, aa in found]
        assert _to_fracs(got, out) == want


def test_table_validation():
    good = _dyadic()
    x = np.ones(8, np.float32)
    oracle.quantize_8bit(x, "f32", 4, good)
    bad = [good[::-1].copy(), np.concatenate([good[:255], good[254:255]]),
           np.where(np.arange(256) == 255, np.float32(1.5), good).astype(np.float32),
           np.where(np.arange(256) == 129, np.float32(1e-30), good).astype(np.float32),
           np.where(np.arange(256) == 3, np.float32("nan"), good).astype(np.float32)]
    for t in bad:
        with pytest.raises(ValueError):
            oracle.quantize_8bit(x, "f32", 4, t)
        with pytest.raises(ValueError):
            oracle.dequantize_8bit(np.zeros(8, np.uint8), np.ones(2, np.float32), 8, 4, t, "f32")


def test_symmetric_pair_decides_tiny_quotients_by_sign():
    """A table whose two smallest entries are -c and +c has a decision threshold
    of exactly 0.  A quotient v = x / absmax far below c is nearer +c when
    positive and -c when negative; a distance taken in float64 (c + |v| and
    c - |v| both rounding to c) would call every such v a tie.  Checked against
    the exact rational restatement, with quotients down to the subnormal range."""
    rng = np.random.default_rng(23)
    c = np.float32(2.0 ** -24)
    vals = {-1.0, 1.0, -float(c), float(c)}
    while len(vals) < 256:
        v = float(np.float32(rng.uniform(-1.0, 1.0)))
        if abs(v) >= 2.0 ** -20:
            vals.add(v)
    code = np.array(sorted(vals), np.float32)
    B = 64
    a = np.float32(1.2680464e-18)
    tiny = np.concatenate([np.float32(a) * np.exp2(-np.arange(30, 120, 6, dtype=np.float64)).astype(np.float32),
                           np.array([1.4e-45, 2.8e-45, 1e-40, 1e-30], np.float32)])
    tiny = tiny[tiny > 0]                          # (the deepest scalings underflow)
    x = np.zeros(B, np.float32)
    x[0] = a
    x[1:1 + tiny.size] = tiny
    x[1 + tiny.size:1 + 2 * tiny.size] = -tiny
    x[2 * tiny.size + 1] = -0.0
    q, _ = oracle.quantize_8bit(x, "f32", B, code)
    codes = [Fraction(float(v)) for v in code]
    idxs, _ = bf.quantize_with_table([Fraction(float(v)) for v in x], B, codes)
    assert list(q) == idxs
    k = int(np.searchsorted(code, 0.0))            # index of +c
    assert all(i == k for i in q[1:1 + tiny.size]) and all(i == k - 1 for i in q[1 + tiny.size:1 + 2 * tiny.size])
