"""quantize_8bit / dequantize_8bit on the GPU against the CPU oracle: bit-exact.

"Feat/mps gemm 4bit bf16", What runs natively now (quantize_blockwise /
dequantize_blockwise) and Correctness (exact nearest code).  The table is the
caller's (the pages print none): tables with evenly spread, log-spread and
clustered entries, and a dyadic linear one.
"""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_b200 as bnb4
import oracle
import synthetic

from gpu_util import to_dev, to_host

pytestmark = pytest.mark.gpu


def _table(kind: str, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    if kind == "dyadic":
        return ((np.arange(256) - 128) / 128.0).astype(np.float32)
    vals = {-1.0, 0.0, 1.0}
    while len(vals) < 256:
        if kind == "uniform":
            v = rng.uniform(-1.0, 1.0)
        elif kind == "log":
            v = rng.choice([-1.0, 1.0]) * 2.0 ** rng.uniform(-24.0, 0.0)
        else:  # clustered near 0
            v = rng.uniform(-1e-3, 1e-3)
        v = float(np.float32(v))
        if v == 0.0 or abs(v) >= 2.0 ** -24:
            vals.add(v)
    return np.array(sorted(vals), np.float32)


def _same16(a, b):
    return np.array_equal(a.view(np.uint32 if a.dtype == np.float32 else np.uint16),
                          b.view(np.uint32 if b.dtype == np.float32 else np.uint16))


@pytest.mark.parametrize("kind", ["uniform", "log", "clustered", "dyadic"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("B", [64, 256, 1024, 4096])
@pytest.mark.parametrize("n", [1, 15, 17, 4096, 3 * 4096 + 77, 100003])
def test_roundtrip_matches_oracle(kind, dtype, B, n):
    code = _table(kind, seed=B + n % 13)
    x = synthetic.roundtrip_tensor(n, seed=n % 97 + B, dtype=dtype)
    xs = synthetic.storage_numpy(x)
    gq, ga = bnb4.quantize_8bit(to_dev(xs, dtype), code, B)
    oq, oa = oracle.quantize_8bit(xs, dtype, B, code)
    assert np.array_equal(to_host(ga).view(np.uint32), oa.view(np.uint32)), "absmax"
    bad = np.nonzero(to_host(gq) != oq)[0]
    assert bad.size == 0, (bad.size, bad[:4])
    for out in ("f32", "f16", "bf16"):
        gd = to_host(bnb4.dequantize_8bit(torch.from_numpy(oq).cuda(), torch.from_numpy(oa).cuda(), code, B,
                                          dtype=synthetic.TORCH_DTYPES[out]))
        assert _same16(gd, oracle.dequantize_8bit(oq, oa, n, B, code, out)), out


@pytest.mark.parametrize("kind", ["uniform", "log", "dyadic"])
def test_midpoint_neighbourhoods(kind):
    """Values at and next to every exact midpoint, in blocks whose absmax is 1."""
    code = _table(kind, seed=3)
    mids = (code[:-1].astype(np.float64) + code[1:].astype(np.float64)) / 2
    m32 = mids.astype(np.float32)
    vs = [m32]
    a, b = m32, m32
    for _ in range(3):
        a, b = np.nextafter(a, np.float32(-2)), np.nextafter(b, np.float32(2))
        vs += [a, b]
    v = np.concatenate(vs)
    v = v[np.abs(v) <= 1.0]
    B = 64
    nb = -(-v.size // (B - 1))
    x = np.zeros(nb * B, np.float32)
    x[0::B] = 1.0
    x[np.nonzero(np.arange(nb * B) % B != 0)[0][:v.size]] = v
    gq, ga = bnb4.quantize_8bit(torch.from_numpy(x).cuda(), code, B)
    oq, oa = oracle.quantize_8bit(x, "f32", B, code)
    assert np.array_equal(to_host(ga), oa)
    bad = np.nonzero(to_host(gq) != oq)[0]
    assert bad.size == 0, (bad.size, x[bad[:4]])


def test_special_values():
    code = _table("uniform", seed=4)
    B = 64
    x = synthetic.normal((B * 6,), 5, 1.0, "f32").numpy().copy()
    x[:B] = 0.0                       # all-zero block
    x[B:2 * B] = -0.0
    x[2 * B + 3] = np.nan             # NaN: skipped by the maximum, index 0
    x[3 * B + 1] = np.inf             # absmax inf: finite -> 0, inf -> NaN -> index 0
    x[4 * B:5 * B] = np.float32(1e-40) * np.arange(1, B + 1)  # subnormal block
    gq, ga = bnb4.quantize_8bit(torch.from_numpy(x).cuda(), code, B)
    oq, oa = oracle.quantize_8bit(x, "f32", B, code)
    assert np.array_equal(to_host(gq), oq)
    assert np.array_equal(to_host(ga).view(np.uint32), oa.view(np.uint32))


def test_full_size_sample():
    """2^22 bf16 elements at blocksize 64 (4 M of the 2^28 round-trip workload)."""
    code = _table("log", seed=8)
    n = 1 << 22
    xs = synthetic.storage_numpy(synthetic.roundtrip_tensor(n, 0, "bf16"))
    gq, ga = bnb4.quantize_8bit(to_dev(xs, "bf16"), code, 64)
    oq, oa = oracle.quantize_8bit(xs, "bf16", 64, code)
    assert np.array_equal(to_host(ga), oa) and np.array_equal(to_host(gq), oq)
    gd = to_host(bnb4.dequantize_8bit(gq, ga, code, 64, dtype=torch.bfloat16))
    assert _same16(gd, oracle.dequantize_8bit(oq, oa, n, 64, code, "bf16"))


def _straddle_table(symmetric: bool) -> np.ndarray:
    """Entries spread over [-1, 1] with no 0 and the two smallest magnitudes
    straddling it: -2^-24 and +2^-24 give a threshold of exactly 0, -2^-24 and
    the float after 2^-24 one of 2^-48 (the smallest a table can have)."""
    rng = np.random.default_rng(21)
    lo = np.float32(2.0 ** -24)
    hi = lo if symmetric else np.nextafter(lo, np.float32(1))
    vals = {-1.0, 1.0, -float(lo), float(hi)}
    while len(vals) < 256:
        v = float(np.float32(rng.uniform(-1.0, 1.0)))
        if abs(v) >= 2.0 ** -20:
            vals.add(v)
    return np.array(sorted(vals), np.float32)


@pytest.mark.parametrize("kind", ["log", "straddle", "symmetric"])
def test_midpoints_over_the_exponent_range(kind):
    """Values next to every midpoint times absmax, for absmax over the whole
    exponent range (around the limits below which the reciprocal path gives
    way to the division: 2^-96, and the table's own floor), plus elements
    whose quotients are tiny or subnormal next to thresholds of 0 and 2^-48."""
    code = _table("log", seed=5) if kind == "log" else _straddle_table(kind == "symmetric")
    mids = (code[:-1].astype(np.float64) + code[1:].astype(np.float64)) / 2
    rng = np.random.default_rng(17)
    exps = np.concatenate([[-126, -120, -100, -97, -96, -95, -80, -60, -54, -53, -52, -51, -30, -1, 0,
                            40, 95, 96, 97, 126, 127], rng.integers(-126, 128, 27)])
    a_all = (rng.uniform(1.0, 2.0, exps.size) * np.exp2(exps.astype(np.float64))).astype(np.float32)
    a_all = a_all[np.isfinite(a_all)]
    B = 64
    blocks = []
    for a in a_all:
        x0 = (mids * np.float64(a)).astype(np.float32)
        cand = [x0]
        up, dn = x0, x0
        for _ in range(3):
            up, dn = np.nextafter(up, np.float32(np.inf)), np.nextafter(dn, np.float32(-np.inf))
            cand += [up, dn]
        tiny = np.float32(a) * np.exp2(-np.arange(40, 160, 4, dtype=np.float64)).astype(np.float32)
        c = np.concatenate(cand + [tiny, -tiny])
        c = c[np.isfinite(c) & (np.abs(c) <= a)]
        for j in range(0, c.size, B - 1):
            blk = np.zeros(B, np.float32)
            blk[0] = a
            part = c[j:j + B - 1]
            blk[1:1 + part.size] = part
            blocks.append(blk)
    x = np.concatenate(blocks)
    gq, ga = bnb4.quantize_8bit(torch.from_numpy(x).cuda(), code, B)
    oq, oa = oracle.quantize_8bit(x, "f32", B, code)
    assert np.array_equal(to_host(ga).view(np.uint32), oa.view(np.uint32))
    bad = np.nonzero(to_host(gq) != oq)[0]
    assert bad.size == 0, (bad.size, x[bad[:4]], x[(bad[:4] // B) * B])
