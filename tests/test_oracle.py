"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: values the
pages or the workload definition print (tests/golden), closed forms,
invariants, an exact rational restatement on tiny inputs (oracle.bruteforce),
or a library routine (torch / numpy conversions, numpy float64 matmul).
"""
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import bruteforce as bf
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = {}
    vals = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                rows[k.strip()] = v.split()
            else:
                vals.append(line)
    return rows, vals


def _to_fracs(arr, dtype):
    if dtype == "f32":
        return [Fraction(float(v)) for v in arr]
    conv = bf.f16_bits_to_fraction if dtype == "f16" else bf.bf16_bits_to_fraction
    return [conv(int(v)) for v in arr]


# ------------------------------------------------------------------ tables

def test_nf4_table_matches_golden_literals_and_invariants():
    _, lits = _read_golden("nf4_table.txt")
    t = oracle.code_table("nf4")
    want = np.array([float(bf.round_to(Fraction(s), "f32")) for s in lits], np.float32)
    assert np.array_equal(t, want)
    assert np.all(np.diff(t) > 0), "NF4 codes ascend strictly"
    assert t[0] == -1.0 and t[15] == 1.0 and t[7] == 0.0
    assert int((t < 0).sum()) == 7 and int((t > 0).sum()) == 8
    gaps = np.diff(t.astype(np.float64))
    assert 0.0795 < gaps.min() < 0.0797 and 0.3037 < gaps.max() < 0.3039


def test_fp4_table_closed_form():
    t = oracle.code_table("fp4")
    # E2M1 magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 scaled by 1/6
    mags = [0, 1 / 12, 1 / 6, 1 / 4, 1 / 3, 1 / 2, 2 / 3, 1]
    for i, m in enumerate(mags):
        assert t[i] == np.float32(m)
        assert t[8 + i] == -np.float32(m)
    assert np.all(np.diff(t[:8]) > 0)
    assert math.copysign(1.0, float(t[8])) == -1.0 and t[8] == 0.0, "index 8 is -0.0"
    assert [float(v) for v in t] == [float(v) for v in bf.fp4_table()]


# ------------------------------------------------------------- conversions

def test_16bit_to_f32_exhaustive_against_torch():
    bits = np.arange(65536, dtype=np.uint16)
    for dtype, tdt in (("f16", torch.float16), ("bf16", torch.bfloat16)):
        ours = oracle.to_f32(bits, dtype)
        ref = torch.from_numpy(bits.view(np.int16)).view(tdt).float().numpy()
        fin = np.isfinite(ref)
        assert np.array_equal(ours[fin].view(np.uint32), ref[fin].view(np.uint32))
        assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_f32_to_16bit_rne_against_torch_and_numpy():
    rng = np.random.default_rng(0)
    # random bit patterns over the whole finite range plus the rounding edges
    b = rng.integers(0, 2**32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    x = b.view(np.float32)
    x = x[np.isfinite(x)]
    edges = []
    for hb in range(0, 65536, 7):
        base = np.uint32(hb) << np.uint32(16)
        for low in (0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x0001):
            edges.append(np.uint32(base | np.uint32(low)))
    e = np.array(edges, np.uint32).view(np.float32)
    x = np.concatenate([x, e[np.isfinite(e)],
                        np.array([65504, 65519.99, 65520, 65536, 6.1e-5, 5.96e-8, 2.98e-8,
                                  2.99e-8, 1e-45, -0.0, 0.0], np.float32)])
    ours_bf = oracle.from_f32(x, "bf16")
    ref_bf = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    fin = np.isfinite(torch.from_numpy(x).to(torch.bfloat16).float().numpy())
    assert np.array_equal(ours_bf[fin], ref_bf[fin])
    ours_h = oracle.from_f32(x, "f16")
    with np.errstate(over="ignore"):
        ref_h = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours_h, ref_h)


# ---------------------------------------------------------------- quantize

def test_worked_example_golden():
    rows, _ = _read_golden("worked_example.txt")
    x = np.array([float(v) for v in rows["x"]], np.float32)
    for q in ("nf4", "fp4"):
        packed, absmax = oracle.quantize(x, "f32", 64, q)
        assert absmax.tolist() == [float(rows["absmax"][0])]
        assert packed.tolist() == [int(h, 16) for h in rows[f"{q}_packed"]]
        _, _, idxs = bf.quantize([Fraction(float(v)) for v in x], 64, q)
        assert idxs == [int(i) for i in rows[f"{q}_idx"]]


def _tiny_inputs():
    cases = []
    rnd = random.Random(1234)
    for dtype in ("f32", "f16", "bf16"):
        for n, B in ((1, 64), (2, 64), (63, 64), (64, 64), (65, 64), (130, 64), (257, 128),
                     (300, 256)):
            cases.append((dtype, n, B, rnd.randrange(1 << 30)))
    return cases


@pytest.mark.parametrize("dtype,n,B,seed", _tiny_inputs())
@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
def test_quantize_matches_exact_bruteforce(dtype, n, B, seed, qtype):
    x = synthetic.normal((n,), seed, 1.0, dtype, outlier_frac=0.05)
    xs = synthetic.storage_numpy(x)
    packed, absmax = oracle.quantize(xs, dtype, B, qtype)
    fr = _to_fracs(xs, dtype)
    bpacked, babsmax, bidx = bf.quantize(fr, B, qtype)
    assert packed.tolist() == bpacked
    assert [Fraction(float(a)) for a in absmax] == babsmax
    # dequantize: oracle vs exact rounding of the fp32 product
    for out in ("f32", "f16", "bf16"):
        d = oracle.dequantize(packed, absmax, n, B, qtype, out)
        want = bf.dequantize(bidx, babsmax, B, qtype, out)
        assert _to_fracs(d, out) == want


@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
def test_ties_go_to_smallest_index(qtype):
    """v exactly on a representable midpoint between two codes: smallest index wins."""
    codes = bf.table(qtype)
    vals = sorted(set(codes))
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    mids = [m for m in mids if bf.round_to(m, "f32") == m]
    assert mids, "at least one representable midpoint"
    # one block: 1.0 fixes absmax = 1 so v == x exactly
    x = np.array([1.0] + [float(m) for m in mids], np.float32)
    packed, absmax = oracle.quantize(x, "f32", 64, qtype)
    assert absmax[0] == 1.0
    got = []
    for i in range(len(x)):
        byte = int(packed[i // 2])
        got.append(byte >> 4 if i % 2 == 0 else byte & 15)
    for m, idx in zip(mids, got[1:]):
        cands = [i for i, c in enumerate(codes) if abs(c - m) == min(abs(c2 - m) for c2 in codes)]
        assert len(cands) >= 2
        assert idx == min(cands)
    if qtype == "fp4":
        assert 8 not in got, "quantize never emits -0 (index 8)"


def test_special_blocks():
    # all-zero block, -0.0, odd tail, +-absmax elements
    x = np.zeros(64 + 3, np.float32)
    x[64] = -3.5
    x[65] = 3.5
    x[66] = -0.0
    for q, zero_idx, pos1, neg1 in (("nf4", 7, 15, 0), ("fp4", 0, 7, 15)):
        packed, absmax = oracle.quantize(x, "f32", 64, q)
        assert absmax.tolist() == [0.0, 3.5]
        assert packed[:32].tolist() == [zero_idx << 4 | zero_idx] * 32
        assert packed[32] == (neg1 << 4) | pos1
        assert packed[33] == zero_idx << 4, "odd tail: low nibble 0"
        d = oracle.dequantize(packed, absmax, x.size, 64, q, "f32")
        assert d[64] == -3.5 and d[65] == 3.5
        assert np.all(d[:64] == 0) and not np.any(np.signbit(d[:64])), "zeros round-trip to +0"
        assert d[66] == 0 and not np.signbit(d[66])


def _bracket_gap(v, codes):
    vals = sorted(set(float(c) for c in codes))
    for a, b in zip(vals, vals[1:]):
        if a <= v <= b:
            return b - a
    raise AssertionError(v)


@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("B", [64, 256, 4096])
def test_error_bound_and_idempotence(qtype, dtype, B):
    n = 3 * B + 17
    x = synthetic.roundtrip_tensor(n, seed=B + len(dtype), dtype=dtype)
    xs = synthetic.storage_numpy(x)
    packed, absmax = oracle.quantize(xs, dtype, B, qtype)
    d = oracle.dequantize(packed, absmax, n, B, qtype, dtype)
    xf = oracle.to_f32(xs, dtype).astype(np.float64)
    df = oracle.to_f32(d, dtype).astype(np.float64)
    codes = oracle.code_table(qtype)
    eps_out = {"f32": 2.0**-24, "f16": 2.0**-11, "bf16": 2.0**-8}[dtype]
    for i in range(n):
        a = float(absmax[i // B])
        v = xf[i] / a
        gap = _bracket_gap(v, codes)
        bound = a * (0.5 * gap + 2.0**-24) + abs(df[i]) * (2.0**-24 + eps_out) + 1e-300
        assert abs(df[i] - xf[i]) <= bound, (i, xf[i], df[i], bound)
    # the +-absmax element of every block round-trips exactly
    for b in range(absmax.size):
        blk = xf[b * B:(b + 1) * B]
        j = int(np.argmax(np.abs(blk)))
        assert df[b * B + j] == blk[j]
    # idempotence: re-quantizing the dequantized tensor reproduces bytes and absmax
    p2, a2 = oracle.quantize(d, dtype, B, qtype)
    assert np.array_equal(p2, packed) and np.array_equal(a2, absmax)


# ------------------------------------------------------------------ matmul

def _quant_weight(N, K, B, qtype, seed=0, sigma=0.02):
    w = synthetic.weight(N, K, seed, sigma).numpy()
    return oracle.quantize(w.reshape(-1), "f32", B, qtype)


def test_matmul_one_hot_gives_weight_column():
    N, K, B = 8, 128, 64
    packed, absmax = _quant_weight(N, K, B, "nf4")
    wdeq = oracle.dequantize(packed, absmax, N * K, B, "nf4", "f32").reshape(N, K)
    for k in (0, 1, 63, 64, 127):
        x = np.zeros(K, np.float32)
        x[k] = 1.0
        xb = oracle.from_f32(x, "bf16")
        y = oracle.matmul(xb, "bf16", packed, absmax, None, 1, N, K, B, "nf4")
        assert np.array_equal(y[0], wdeq[:, k].astype(np.float64))


def test_matmul_constant_blocks_closed_form():
    """Every block constant and positive: all codes are +1, so y_j = sum_b B * a_b."""
    N, K, B = 4, 256, 64
    rng = np.random.default_rng(7)
    a = rng.uniform(0.5, 2.0, size=(N, K // B)).astype(np.float32)
    w = np.repeat(a, B, axis=1)
    for q in ("nf4", "fp4"):
        packed, absmax = oracle.quantize(w.reshape(-1), "f32", B, q)
        assert np.array_equal(absmax.reshape(N, -1), a)
        x = oracle.from_f32(np.ones(K, np.float32), "f16")
        y = oracle.matmul(x, "f16", packed, absmax, None, 1, N, K, B, q)
        want = (B * a.astype(np.float64)).sum(axis=1)
        assert np.allclose(y[0], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
def test_matmul_and_backward_exact_bruteforce(qtype):
    _matmul_and_backward_exact(qtype, "bf16")


@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
def test_matmul_and_backward_exact_bruteforce_fp32_activations(qtype):
    """The fp32 compute dtype: fp32 activations, bias and gradients."""
    _matmul_and_backward_exact(qtype, "f32")


def _matmul_and_backward_exact(qtype, dt):
    M, N, K, B = 3, 64, 128, 64
    packed, absmax = _quant_weight(N, K, B, qtype, seed=5)
    X = synthetic.activations(M, K, seed=6, dtype=dt)
    Xs = synthetic.storage_numpy(X).reshape(-1)
    bias = synthetic.storage_numpy(synthetic.bias(N, seed=8, dtype=dt))
    dY = synthetic.storage_numpy(synthetic.grad_output(M, N, seed=9, dtype=dt)).reshape(-1)
    # exact weights from the brute force
    idx = []
    for byte in packed.tolist():
        idx += [byte >> 4, byte & 15]
    idx = idx[:N * K]
    wq = bf.dequantize(idx, [Fraction(float(a)) for a in absmax], B, qtype, "f32")
    W = [wq[j * K:(j + 1) * K] for j in range(N)]
    Xf = [_to_fracs(Xs[m * K:(m + 1) * K], dt) for m in range(M)]
    bfr = _to_fracs(bias, dt)
    Yex = bf.matmul(Xf, W, bfr)
    Y = oracle.matmul(Xs, dt, packed, absmax, bias, M, N, K, B, qtype)
    for m in range(M):
        for j in range(N):
            assert abs(Y[m, j] - float(Yex[m][j])) <= 1e-12 * (1 + abs(float(Yex[m][j])))
    # backward: dX = dY @ W (reduction over N) -- exact, then the entries form
    dYf = [_to_fracs(dY[m * N:(m + 1) * N], dt) for m in range(M)]
    WT = [[W[j][k] for j in range(N)] for k in range(K)]
    dXex = bf.matmul(dYf, WT)
    dX = oracle.matmul_backward(dY, dt, packed, absmax, M, N, K, B, qtype)
    for m in range(M):
        for k in range(K):
            assert abs(dX[m, k] - float(dXex[m][k])) <= 1e-12 * (1 + abs(float(dXex[m][k])))
    ms = np.array([0, 2, 1, 2])
    ks = np.array([0, 127, 64, 5])
    assert np.array_equal(
        oracle.matmul_backward_entries(dY, dt, packed, absmax, M, N, K, B, qtype, ms, ks),
        dX[ms, ks])
    js = np.array([63, 0, 17, 32])
    assert np.array_equal(
        oracle.matmul_entries(Xs, dt, packed, absmax, bias, M, N, K, B, qtype, ms, js),
        Y[ms, js])


def test_backward_is_transposed_forward_against_numpy():
    """dX = dY @ Wdeq; checked with numpy's float64 matmul on the dequantized weight."""
    M, N, K, B = 5, 96, 192, 64
    packed, absmax = _quant_weight(N, K, B, "nf4", seed=11)
    wdeq = oracle.dequantize(packed, absmax, N * K, B, "nf4", "f32").reshape(N, K)
    dY = synthetic.storage_numpy(synthetic.grad_output(M, N, seed=12, dtype="f16"))
    dYf = oracle.to_f32(dY, "f16").reshape(M, N).astype(np.float64)
    dX = oracle.matmul_backward(dY, "f16", packed, absmax, M, N, K, B, "nf4")
    assert np.allclose(dX, dYf @ wdeq.astype(np.float64), rtol=1e-12, atol=1e-12)
    X = synthetic.storage_numpy(synthetic.activations(M, K, seed=13, dtype="f16"))
    Xf = oracle.to_f32(X, "f16").reshape(M, K).astype(np.float64)
    Y = oracle.matmul(X, "f16", packed, absmax, None, M, N, K, B, "nf4")
    assert np.allclose(Y, Xf @ wdeq.astype(np.float64).T, rtol=1e-12, atol=1e-12)


def test_oracle_rejects_bad_arguments():
    x = np.zeros(8, np.float32)
    with pytest.raises(ValueError):
        oracle.quantize(x, "f32", 0, "nf4")
    with pytest.raises(TypeError):
        oracle.quantize(x.astype(np.float64), "f32", 64, "nf4")


# ------------------------------------------------------- knife-edge inputs

@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
def test_division_knife_edges_match_exact_quotient(qtype):
    """Blocks where x/a and x*fp32(1/a) choose different codes: the oracle follows x/a."""
    import adversarial
    blk = adversarial.division_blocks(qtype, 64)
    assert blk.size >= 64 * 20
    packed, absmax = oracle.quantize(blk, "f32", 64, qtype)
    bpacked, babsmax, _ = bf.quantize([Fraction(float(v)) for v in blk], 64, qtype)
    assert packed.tolist() == bpacked


@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
@pytest.mark.parametrize("out", ["bf16", "f16"])
def test_dequant_double_rounding_edges(qtype, out):
    """Pairs where rounding the exact product straight to 16 bits would differ."""
    import adversarial
    pairs = adversarial.double_rounding_pairs(qtype, out)
    assert len(pairs) >= 4
    n = 2 * len(pairs)
    packed = np.zeros(len(pairs), np.uint8)
    absmax = np.zeros(len(pairs), np.float32)
    for i, (ci, a) in enumerate(pairs):
        packed[i] = (ci << 4) | ci
        absmax[i] = a
    d = oracle.dequantize(packed, absmax, n, 2, qtype, out)
    want = bf.dequantize([ci for ci, _ in pairs for _ in (0, 1)],
                         [Fraction(float(a)) for a in absmax], 2, qtype, out)
    assert _to_fracs(d, out) == want
