"""quantize_4bit / dequantize_4bit on the GPU against the CPU oracle: bit-exact."""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_b200 as bnb4
import oracle
import synthetic

from gpu_util import to_dev, to_host, unpack_nibbles

pytestmark = pytest.mark.gpu

BLOCKSIZES = [64, 128, 256, 512, 1024, 2048, 4096]
DTYPES = ["f32", "f16", "bf16"]


def _gpu_quant(xs, dtype, B, q):
    packed, absmax = bnb4.quantize_4bit(to_dev(xs, dtype), B, q)
    return to_host(packed), to_host(absmax)


def _gpu_dequant(packed, absmax, n, B, q, out):
    t = bnb4.dequantize_4bit(torch.from_numpy(packed).cuda(), torch.from_numpy(absmax).cuda(),
                             n, B, q, dtype=synthetic.TORCH_DTYPES[out])
    return to_host(t)


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("B", BLOCKSIZES)
@pytest.mark.parametrize("n", [1, 15, 17, 4096, 3 * 4096 + 77, 100003])
def test_roundtrip_matches_oracle(q, dtype, B, n):
    x = synthetic.roundtrip_tensor(n, seed=n % 97 + B, dtype=dtype)
    xs = synthetic.storage_numpy(x)
    gp, ga = _gpu_quant(xs, dtype, B, q)
    op, oa = oracle.quantize(xs, dtype, B, q)
    assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32)), "absmax"
    assert np.array_equal(gp, op), "packed bytes"
    for out in DTYPES:
        gd = _gpu_dequant(op, oa, n, B, q, out)
        od = oracle.dequantize(op, oa, n, B, q, out)
        assert np.array_equal(gd.view(np.uint32 if out == "f32" else np.uint16),
                              od.view(np.uint32 if out == "f32" else np.uint16)), out


@pytest.mark.parametrize("q", ["nf4", "fp4"])
def test_division_knife_edges(q):
    """Blocks where x/a and x*fp32(1/a) pick different codes."""
    import adversarial
    blk = adversarial.division_blocks(q, 64, seed=3, per_threshold=4)
    gp, ga = _gpu_quant(blk, "f32", 64, q)
    op, oa = oracle.quantize(blk, "f32", 64, q)
    assert np.array_equal(gp, op) and np.array_equal(ga, oa)


@pytest.mark.parametrize("q", ["nf4", "fp4"])
def test_quotients_next_to_every_threshold(q):
    """x within 4 fp32 steps of every decision threshold times a, for 2048 absmax
    values over the whole exponent range (both sides of the reciprocal path's
    range limits included)."""
    import adversarial
    blk = adversarial.threshold_neighbourhoods(q, 64, n_scales=2048, radius=4, seed=11)
    gp, ga = _gpu_quant(blk, "f32", 64, q)
    op, oa = oracle.quantize(blk, "f32", 64, q)
    assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32))
    bad = np.nonzero(gp != op)[0]
    assert bad.size == 0, (bad.size, bad[:4])


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("out", ["bf16", "f16"])
def test_dequant_double_rounding_edges(q, out):
    import adversarial
    pairs = adversarial.double_rounding_pairs(q, out, want=16)
    packed = np.array([(ci << 4) | ci for ci, _ in pairs], np.uint8)
    absmax = np.array([a for _, a in pairs], np.float32)
    # one 64-element block per pair: repeat each byte over its block
    packed64 = np.repeat(packed, 32)
    n = packed64.size * 2
    gd = _gpu_dequant(packed64, absmax, n, 64, q, out)
    od = oracle.dequantize(packed64, absmax, n, 64, q, out)
    assert np.array_equal(gd, od)


def test_special_values():
    # all-zero block, +-absmax, -0.0, odd tail, subnormal and huge absmax
    x = np.zeros(64 * 6 + 3, np.float32)
    x[64:128] = np.linspace(-3.5, 3.5, 64, dtype=np.float32)
    x[128:192] = np.float32(1e-40) * np.arange(64, dtype=np.float32)     # subnormal absmax
    x[192:256] = np.float32(3e38) * np.linspace(-1, 1, 64, dtype=np.float32)  # near overflow
    x[256:320] = -0.0
    x[320:384] = np.float32(2.0**-100) * np.linspace(-1, 1, 64, dtype=np.float32)
    x[-3:] = [1.0, -0.5, 0.25]
    for q in ("nf4", "fp4"):
        gp, ga = _gpu_quant(x, "f32", 64, q)
        op, oa = oracle.quantize(x, "f32", 64, q)
        assert np.array_equal(gp, op) and np.array_equal(ga.view(np.uint32), oa.view(np.uint32))
        assert gp[-1] & 15 == 0, "odd tail keeps the low nibble 0"


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("q", ["nf4", "fp4"])
def test_nan_and_inf_elements(q, dtype):
    """NaN is skipped by the maximum and gets index 0; an infinite element makes
    absmax infinite, so the block's finite elements normalise to 0 and the
    infinite ones to NaN (index 0)."""
    tdt = synthetic.TORCH_DTYPES[dtype]
    x = synthetic.roundtrip_tensor(64 * 40 + 9, seed=17, dtype=dtype).float()
    x[5] = float("nan")                     # a NaN among ordinary values
    x[64 * 3: 64 * 4: 7] = float("nan")     # several in one block
    x[64 * 6: 64 * 7] = float("nan")        # a block of NaN only: absmax 0
    x[64 * 9 + 3] = float("inf")
    x[64 * 12 + 60] = -float("inf")
    x[64 * 15 + 1] = float("nan")
    x[64 * 15 + 2] = float("inf")
    x[-4] = float("nan")                    # in the ragged tail
    xs = synthetic.storage_numpy(x.to(tdt))
    for B in (64, 256):
        gp, ga = _gpu_quant(xs, dtype, B, q)
        op, oa = oracle.quantize(xs, dtype, B, q)
        assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32)), ("absmax", B)
        bad = np.nonzero(gp != op)[0]
        assert bad.size == 0, (B, bad.size, bad[:4])


def _fp4_ratio_ties(n, B, dtype, seed):
    """Blocks whose elements are the block's absmax times each FP4 decision point
    k / 24, rounded to the input dtype (often exact: x / a lands on the point),
    with a third of them moved one step of the dtype either way, random signs,
    absmax over a wide exponent range, zeros and a NaN in some blocks."""
    tdt = synthetic.TORCH_DTYPES[dtype]
    g = torch.Generator().manual_seed(seed)
    nb = -(-n // B)
    lo, hi = (-40, 40) if dtype == "bf16" else (-12, 12)
    a = ((torch.rand(nb, generator=g) * 4 + 0.25) * 2.0 ** torch.randint(lo, hi, (nb,), generator=g).float())
    a = a.to(tdt).float()
    k = torch.tensor([0, 1, 3, 5, 7, 10, 14, 20, 24], dtype=torch.float32)
    x = (a[:, None] * k[torch.randint(0, len(k), (nb, B), generator=g)] / 24).to(tdt)
    step = torch.randint(-1, 2, (nb, B), generator=g).to(torch.int16)
    moved = (x.view(torch.int16) + step).view(tdt)
    x = torch.where((torch.rand(nb, B, generator=g) < 0.3) & (x != 0), moved, x)
    x = x * torch.where(torch.rand(nb, B, generator=g) < 0.5, -1.0, 1.0).to(tdt)
    x[:, 0] = a.to(tdt)
    nan_blocks = torch.rand(nb, generator=g) < 0.05
    x[nan_blocks, B // 2] = float("nan")
    return synthetic.storage_numpy(x.reshape(-1)[:n].contiguous())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("B", [64, 256, 4096])
@pytest.mark.parametrize("n", [64, 4096 * 3 + 17, 1 << 20])
def test_fp4_exact_ratio_ties(dtype, B, n):
    """FP4 decision points are short fractions k / 24 that ratios of 16-bit
    inputs hit exactly (and otherwise stay clear of by a fixed gap); each tie
    must go where the IEEE quotient sends it."""
    xs = _fp4_ratio_ties(n, B, dtype, seed=n % 101 + B)
    gp, ga = _gpu_quant(xs, dtype, B, "fp4")
    op, oa = oracle.quantize(xs, dtype, B, "fp4")
    assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32)), "absmax"
    bad = np.nonzero(gp != op)[0]
    assert bad.size == 0, (bad.size, bad[:4])


def test_n_zero_is_a_noop():
    packed, absmax = bnb4.quantize_4bit(torch.empty(0, device="cuda"), 64, "nf4")
    assert packed.numel() == 0 and absmax.numel() == 0


def _transitions(q):
    """Oracle code as a step function of v >= 0 and v <= 0 over fp32 bit patterns."""
    def code_of(bits_u32, sign):
        v = np.array([bits_u32], np.uint32).view(np.float32) * (-1 if sign else 1)
        p, _ = oracle.quantize(np.array([1.0, v[0]], np.float32), "f32", 64, q)
        return int(p[0]) & 15
    one = 0x3F800000
    out = {}
    for sign in (0, 1):
        pts = []  # (first bits value with this code)
        lo_code = code_of(0, sign)
        pts.append((0, lo_code))
        cur = 0
        while True:
            c = code_of(cur, sign)
            # find the first bits > cur whose code differs, by bisection on [cur, one]
            if code_of(one, sign) == c:
                break
            lo, hi = cur, one
            while hi - lo > 1:
                mid = (lo + hi) // 2
                if code_of(mid, sign) == c:
                    lo = mid
                else:
                    hi = mid
            pts.append((hi, code_of(hi, sign)))
            cur = hi
        out[sign] = pts
    return out


@pytest.mark.parametrize("q", ["nf4", "fp4"])
def test_every_fp32_v_in_unit_interval(q):
    """All 2 * (2^30 + 2^23 + 1) fp32 values v in [-1, 1]: GPU code == oracle code.

    Each 4096-element block is [1.0, 4095 test values], so v = x exactly.  The
    oracle's code, a step function of v, is read off at its transition points
    (found by bisection with the oracle); the comparison runs on the device.
    """
    trans = _transitions(q)
    one = 0x3F800000
    chunk = 4095 * (1 << 16)
    for sign in (0, 1):
        starts = torch.tensor([b for b, _ in trans[sign]], dtype=torch.int64, device="cuda")
        codes = torch.tensor([c for _, c in trans[sign]], dtype=torch.uint8, device="cuda")
        for c0 in range(0, one + 1, chunk):
            bits = torch.arange(c0, min(one + 1, c0 + chunk), dtype=torch.int64, device="cuda")
            m = bits.numel()
            nb = (m + 4094) // 4095
            vals = bits.to(torch.int32).view(torch.float32)
            if sign:
                vals = -vals
            body = torch.zeros(nb * 4095, dtype=torch.float32, device="cuda")
            body[:m] = vals
            x = torch.ones(nb, 4096, dtype=torch.float32, device="cuda")
            x[:, 1:] = body.view(nb, 4095)
            packed, absmax = bnb4.quantize_4bit(x.view(-1), 4096, q)
            nib = torch.stack([packed >> 4, packed & 15], dim=1).view(nb, 4096)[:, 1:]
            got = nib.reshape(-1)[:m]
            want = codes[torch.searchsorted(starts, bits, right=True) - 1]
            bad = torch.nonzero(got != want)
            assert bad.numel() == 0, (sign, hex(int(bits[bad[0, 0]])), int(got[bad[0, 0]]),
                                      int(want[bad[0, 0]]))
            assert bool((absmax == 1.0).all())
            del bits, vals, body, x, packed, absmax, nib, got, want
        torch.cuda.empty_cache()


def _full_blocks_sample(n, B, rng, count=48):
    nb = (n + B - 1) // B
    return np.unique(np.concatenate([[0, nb - 1], rng.integers(0, nb, size=count)]))


@pytest.mark.parametrize("dtype,seeds", [("bf16", [0, 1, 2, 3]), ("f16", [0]), ("f32", [0])])
def test_full_size_2p28_sampled_blocks(dtype, seeds):
    """2^28 elements, N(0,1) with 1% x20 outliers, every quant type and blocksize:
    sampled blocks bit-exact against the oracle; the whole tensor re-quantizes to
    itself (idempotence) and stays inside the error bound."""
    n = 1 << 28
    rng = np.random.default_rng(0)
    for seed in seeds:
        x = synthetic.roundtrip_tensor(n, seed, dtype)
        xd = x.cuda()
        xs = synthetic.storage_numpy(x)
        del x
        for q in ("nf4", "fp4"):
            for B in BLOCKSIZES:
                packed, absmax = bnb4.quantize_4bit(xd, B, q)
                deq = bnb4.dequantize_4bit(packed, absmax, n, B, q, dtype=xd.dtype)
                p2, a2 = bnb4.quantize_4bit(deq, B, q)
                assert torch.equal(p2, packed) and torch.equal(a2, absmax), "idempotence"
                # half the largest code gap (NF4 0.3038, FP4 1/3) plus output rounding
                half_gap = 0.152 if q == "nf4" else 0.1667
                a_el = absmax.repeat_interleave(B)[:n]
                err = (deq.float() - xd.float()).abs()
                assert bool((err <= (half_gap + 2.0**-7) * a_el).all()), "error bound"
                hp = to_host(packed)
                ha = to_host(absmax)
                hd = to_host(deq)
                for b in _full_blocks_sample(n, B, rng):
                    lo, hi = b * B, min(n, (b + 1) * B)
                    op, oa = oracle.quantize(xs[lo:hi], dtype, B, q)
                    assert np.array_equal(hp[lo // 2:(hi + 1) // 2], op), (seed, q, B, b)
                    assert ha[b] == oa[0]
                    od = oracle.dequantize(op, oa, hi - lo, B, q, dtype)
                    assert np.array_equal(hd[lo:hi], od)
                del packed, absmax, deq, p2, a2, a_el, err
        del xd
        torch.cuda.empty_cache()


def test_full_size_2p28_every_run_whole_tensor_digests():
    """Every run of the full-size round-trip sweep (2^28 elements, seeds 0..3,
    fp32 / fp16 / bf16, NF4 / FP4, blocksizes 64..4096: 168 runs): the SHA-256
    digests of the GPU's packed bytes, absmax and dequantized tensor equal the
    CPU oracle's, stored in tests/golden/roundtrip_2p28_digests.json by
    tests/golden/make_roundtrip_digests.py (which calls only the oracle).  So
    every element of every run is compared, not a sample."""
    import hashlib
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "roundtrip_2p28_digests.json")
    with open(path) as f:
        doc = json.load(f)
    n = doc["n"]

    def digest(t):
        return hashlib.sha256(memoryview(to_host(t)).cast("B")).hexdigest()

    bad = []
    torch_dt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    for seed in doc["seeds"]:
        for dt in doc["dtypes"]:
            x = synthetic.roundtrip_tensor(n, seed, dt).cuda()
            deq = torch.empty(n, dtype=torch_dt[dt], device="cuda")
            for qt in doc["quant_types"]:
                for B in doc["blocksizes"]:
                    packed, absmax = bnb4.quantize_4bit(x, B, qt)
                    bnb4.dequantize_4bit(packed, absmax, n, B, qt, out=deq)
                    want = doc["runs"][f"{dt}/{qt}/B{B}/seed{seed}"]
                    got = {"packed": digest(packed), "absmax": digest(absmax), "dequant": digest(deq)}
                    bad += [(f"{dt}/{qt}/B{B}/seed{seed}", k) for k in got if got[k] != want[k]]
                    del packed, absmax
            del x, deq
    assert len(doc["runs"]) == 168 and not bad, bad[:8]
