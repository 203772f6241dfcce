"""double_quant / dequant_absmax on the GPU against the CPU oracle: bit-exact.

"mps-bitsandbytes 0.4.7", Functional API, Double Quantization: the fp32
absmax array is itself quantized to 8 bits with one fp32 scale per group of
256 (the group size is a parameter).  Every step is one IEEE fp32 operation,
so codes, scales and the inverse match the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_b200 as bnb4
import oracle
import synthetic

from gpu_util import to_host

pytestmark = pytest.mark.gpu

GROUPS = [32, 64, 256, 1024, 4096]


def _same_bits(x: np.ndarray, y: np.ndarray) -> bool:
    """fp32 arrays equal bit for bit, any NaN matching any NaN (IEEE 754 fixes
    no payload: the GPU writes 0x7fffffff where x86 writes 0xffc00000)."""
    eq = (x.view(np.uint32) == y.view(np.uint32)) | (np.isnan(x) & np.isnan(y))
    return bool(eq.all())


def _check(a: np.ndarray, group: int):
    a = np.ascontiguousarray(a, np.float32)
    gq, gs = bnb4.double_quant(torch.from_numpy(a).cuda(), group)
    oq, os_ = oracle.double_quant(a, group)
    gq, gs = to_host(gq), to_host(gs)
    assert _same_bits(gs, os_), "scales"
    bad = np.nonzero(gq != oq)[0]
    assert bad.size == 0, (bad.size, bad[:4], a[bad[:4]])
    # inverse, from the oracle's codes
    gd = to_host(bnb4.dequant_absmax(torch.from_numpy(oq).cuda(), torch.from_numpy(os_).cuda(), group))
    od = oracle.dequant_absmax(oq, os_, group)
    assert _same_bits(gd, od), "dequant_absmax"


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("n", [1, 3, 31, 255, 256, 257, 4096 * 3 + 5, 100003])
def test_matches_oracle(group, n):
    a = synthetic.absmax_values(n, seed=n % 89 + group, zero_frac=0.01).numpy()
    _check(a, group)


@pytest.mark.parametrize("group", [32, 256])
def test_special_values(group):
    """Zero groups, NaN, inf, negatives and -0, subnormals, values that land on
    code midpoints (k + 1/2) / 255 of their group maximum."""
    n = group * 8 + 7
    a = synthetic.absmax_values(n, seed=5).numpy().copy()
    a[:group] = 0.0                                   # all-zero group: scale +0, codes 0
    a[group:2 * group] = -0.0
    a[2 * group + 3] = np.nan                         # NaN: skipped by the maximum, code 0
    a[3 * group:4 * group] = np.nan
    a[4 * group + 1] = np.inf                         # scale inf: finite values -> 0, inf -> NaN -> 0;
    #                                                   the inverse gives 0 * inf = NaN
    a[5 * group + 2] = -1.0                           # negative -> clamp to 0
    a[5 * group + 4] = np.float32(1e-42)              # subnormal
    g6 = 6 * group
    a[g6] = 1.0                                       # the group maximum
    a[g6 + 1:g6 + 33] = ((np.arange(32) + 0.5) / 255).astype(np.float32)
    a[7 * group:8 * group] = np.float32(1e-40) * np.arange(1, group + 1)  # subnormal group
    _check(a, group)


def test_full_size_weight_absmax():
    """The absmax array of a 4096 x 11008 weight in blocks of 64 (704,512 values)."""
    a = synthetic.absmax_values(4096 * 11008 // 64, seed=9).numpy()
    _check(a, 256)


def test_argument_checks():
    a = torch.ones(300, device="cuda")
    q = torch.empty(300, dtype=torch.uint8, device="cuda")
    s = torch.empty(2, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    for bad in (0, 16, 100, 8192):
        assert bnb4.bnb4_double_quant(a.data_ptr(), 300, bad, q.data_ptr(), s.data_ptr(), st) == 3
        assert bnb4.bnb4_dequant_absmax(q.data_ptr(), s.data_ptr(), 300, bad, a.data_ptr(), st) == 3
    assert bnb4.bnb4_double_quant(a.data_ptr(), -1, 256, q.data_ptr(), s.data_ptr(), st) == 4
    assert bnb4.bnb4_double_quant(0, 0, 256, 0, 0, st) == 0        # n == 0: nothing enqueued
    assert bnb4.bnb4_double_quant(0, 5, 256, q.data_ptr(), s.data_ptr(), st) == 1
    assert bnb4.bnb4_double_quant(a.data_ptr() + 4, 5, 256, q.data_ptr(), s.data_ptr(), st) == 2


# ------------------------------------------------- gemv on 8-bit statistics

def _weight(N, K, B, q, seed):
    w = synthetic.weight(N, K, seed, 0.02).numpy().reshape(-1)
    packed, absmax = oracle.quantize(w, "f32", B, q)
    return packed, absmax


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("N,K,B", [(96, 4096, 64), (17, 128, 64), (70, 4672, 64), (33, 512, 128),
                                   (40, 8192, 4096), (300, 2048, 256)])
@pytest.mark.parametrize("group", [32, 256, 4096])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemv_dq_matches_oracle(q, dt, N, K, B, group, with_bias):
    """y = x @ dequant(W)^T (+ bias) with W's absmax rebuilt from its double
    quantization; codes whose words straddle rows and a ragged last word
    (N*K/B not a multiple of 4) included."""
    from gpu_util import MATMUL_TOL, as_f64, rel_l2, to_dev
    packed, absmax = _weight(N, K, B, q, seed=N + K + group)
    aq, asc = oracle.double_quant(absmax, group)
    absmax2 = oracle.dequant_absmax(aq, asc, group)
    xs = synthetic.storage_numpy(synthetic.activations(1, K, seed=1, dtype=dt)).reshape(-1)
    bs = synthetic.storage_numpy(synthetic.bias(N, seed=2, dtype=dt)) if with_bias else None
    db = None if bs is None else to_dev(bs, dt)
    dx, dp = to_dev(xs, dt), torch.from_numpy(packed).cuda()
    y = bnb4.gemv_4bit_dq(dx, dp, torch.from_numpy(aq).cuda(), torch.from_numpy(asc).cuda(), N, K,
                          db, B, q, group)
    ref = oracle.matmul(xs, dt, packed, absmax2, bs, 1, N, K, B, q)[0]
    err = rel_l2(as_f64(to_host(y), dt), ref)
    assert err <= MATMUL_TOL, err
    # the kernel rebuilds absmax exactly: same bits as the fp32-absmax gemv on dequant_absmax's output
    y2 = bnb4.gemv_4bit(dx, dp, torch.from_numpy(absmax2).cuda(), N, K, db, B, q)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 14336), (14336, 4096)])
def test_gemv_dq_llama_decode_shapes_sampled(K, N):
    from gpu_util import MATMUL_TOL, as_f64, rel_l2, to_dev
    packed, absmax = _weight(N, K, 64, "nf4", seed=0)
    aq, asc = oracle.double_quant(absmax, 256)
    absmax2 = oracle.dequant_absmax(aq, asc, 256)
    xs = synthetic.storage_numpy(synthetic.activations(1, K, seed=1)).reshape(-1)
    y = to_host(bnb4.gemv_4bit_dq(to_dev(xs, "bf16"), torch.from_numpy(packed).cuda(),
                                  torch.from_numpy(aq).cuda(), torch.from_numpy(asc).cuda(), N, K))
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(K + N).integers(0, N, 254)]))
    ms = np.zeros(rows.size, np.int64)
    ref = oracle.matmul_entries(xs, "bf16", packed, absmax2, None, 1, N, K, 64, "nf4", ms, rows)
    err = rel_l2(as_f64(y, "bf16")[rows], ref)
    assert err <= MATMUL_TOL, err


def test_gemv_dq_argument_checks():
    st = torch.cuda.current_stream().cuda_stream
    x = torch.zeros(256, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(64 * 128, dtype=torch.uint8, device="cuda")
    aq = torch.zeros(256, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(8, device="cuda")
    y = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    args = lambda **kw: [kw.get("x", x.data_ptr()), w.data_ptr(), kw.get("aq", aq.data_ptr()),
                         kw.get("sc", sc.data_ptr()), kw.get("g", 32), None, y.data_ptr(), 64,
                         kw.get("K", 256), 64, 0, 2, st]
    assert bnb4.bnb4_gemv_dq(*args()) == 0
    assert bnb4.bnb4_gemv_dq(*args(sc=0)) == 1
    assert bnb4.bnb4_gemv_dq(*args(aq=0)) == 1
    assert bnb4.bnb4_gemv_dq(*args(aq=aq.data_ptr() + 4)) == 2
    assert bnb4.bnb4_gemv_dq(*args(g=48)) == 3
    assert bnb4.bnb4_gemv_dq(*args(K=40 * 1024)) == 4
    torch.cuda.synchronize()


def test_dequant_absmax_every_significand():
    """The inverse's step RN(scale / 255) for every fp32 significand (scales in
    [1, 2)), and random significands at the exponents around the kernel's
    fast-division range (2^-101 .. 2^101) and in the subnormals: code 1 gives
    the step itself, codes 255 and 128 its products."""
    G = 32
    rng = np.random.default_rng(7)
    edge = []
    for e in (-126, -102, -101, -100, -99, -60, 60, 99, 100, 101, 126):
        m = rng.integers(0, 1 << 23, 4096, dtype=np.uint32)
        edge.append(((np.uint32(e + 127) << 23) | m).view(np.float32))
    edge.append(rng.integers(1, 1 << 23, 4096, dtype=np.uint32).view(np.float32))  # subnormals
    edge.append(np.array([0.0, np.inf, np.float32(2.0 ** -100), np.float32(2.0 ** 100)], np.float32))
    chunks = [((np.uint32(127) << 23) | np.arange(c << 21, (c + 1) << 21, dtype=np.uint32)).view(np.float32)
              for c in range(4)] + [np.concatenate(edge)]
    for sc in chunks:
        n = sc.size * G
        q = np.zeros(n, np.uint8)
        q[0::G], q[1::G], q[2::G] = 1, 255, 128
        got = to_host(bnb4.dequant_absmax(torch.from_numpy(q).cuda(), torch.from_numpy(sc).cuda(), G))
        want = oracle.dequant_absmax(q, sc, G)
        for o in range(3):
            assert _same_bits(got[o::G], want[o::G]), o


# ------------------------------------------- matmuls with M >= 2 on 8-bit statistics

def _dq_weight(N, K, B, q, group, seed):
    w = synthetic.weight(N, K, seed, 0.02).numpy().reshape(-1)
    packed, absmax = oracle.quantize(w, "f32", B, q)
    dp, da = torch.from_numpy(packed).cuda(), torch.from_numpy(absmax).cuda()
    aq, asc = bnb4.double_quant(da, group)
    back = bnb4.dequant_absmax(aq, asc, group)   # the absmax the 8-bit statistics stand for
    return packed, dp, aq, asc, back


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("M,N,K,B,group", [(2, 96, 2048, 64, 256), (9, 45, 1600, 64, 32),
                                           (16, 64, 4096, 256, 256), (17, 256, 512, 64, 256),
                                           (300, 264, 704, 64, 64), (300, 96, 256, 128, 1024)])
def test_gemm_dq_bit_identical_to_fp32_absmax(q, dt, M, N, K, B, group):
    """gemm_4bit_dq equals gemm_4bit given the absmax dequant_absmax writes, bit
    for bit (small-M and tcgen05 kernels; absmax rows with and without a 16-byte
    pitch), and stays within the matmul bar of the float64 oracle."""
    from gpu_util import MATMUL_TOL, as_f64, rel_l2, to_dev
    packed, dp, aq, asc, back = _dq_weight(N, K, B, q, group, seed=M + N)
    Xs = synthetic.storage_numpy(synthetic.activations(M, K, seed=1, dtype=dt)).reshape(-1)
    X = to_dev(Xs, dt).view(M, K)
    bias = to_dev(synthetic.storage_numpy(synthetic.bias(N, seed=2, dtype=dt)), dt) if M % 2 else None
    Ydq = to_host(bnb4.gemm_4bit_dq(X, dp, aq, asc, N, bias, B, q, group))
    Yref = to_host(bnb4.gemm_4bit(X, dp, back, N, bias, B, q))
    assert np.array_equal(Ydq, Yref)
    bs = None if bias is None else to_host(bias)
    ref = oracle.matmul(Xs, dt, packed, to_host(back), bs, M, N, K, B, q)
    assert rel_l2(as_f64(Ydq, dt).reshape(M, N), ref) <= MATMUL_TOL


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("M,N,K,B,group", [(64, 264, 2048, 128, 256), (130, 520, 768, 64, 32)])
def test_gemm_backward_dq_bit_identical_to_fp32_absmax(q, M, N, K, B, group):
    from gpu_util import MATMUL_TOL, as_f64, rel_l2, to_dev
    packed, dp, aq, asc, back = _dq_weight(N, K, B, q, group, seed=N)
    dYs = synthetic.storage_numpy(synthetic.grad_output(M, N, seed=3)).reshape(-1)
    dY = to_dev(dYs, "bf16").view(M, N)
    got = to_host(bnb4.gemm_4bit_backward_dq(dY, dp, aq, asc, K, B, q, group))
    assert np.array_equal(got, to_host(bnb4.gemm_4bit_backward(dY, dp, back, K, B, q)))
    ref = oracle.matmul_backward(dYs, "bf16", packed, to_host(back), M, N, K, B, q)
    assert rel_l2(as_f64(got, "bf16").reshape(M, K), ref) <= MATMUL_TOL


@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_gemm_dq_70b_shapes_m16_sampled(K, N):
    """M = 16 on the 70B-shaped weights with 8-bit statistics: bit-identical to
    the fp32-absmax kernel on the inverse's absmax (whole output)."""
    from gpu_util import to_dev
    w = synthetic.normal((N * K,), 0, 0.015, "f32", device="cuda")
    dp, da = bnb4.quantize_4bit(w, 64, "nf4")
    del w
    aq, asc = bnb4.double_quant(da, 256)
    back = bnb4.dequant_absmax(aq, asc, 256)
    X = synthetic.normal((16, K), 1, 1.0, "bf16", device="cuda")
    assert torch.equal(bnb4.gemm_4bit_dq(X, dp, aq, asc, N), bnb4.gemm_4bit(X, dp, back, N))


def test_gemm_dq_argument_checks():
    A = 1 << 20
    g = bnb4.bnb4_gemm_dq
    assert g(A, A, A, None, 256, None, A, 4, 64, 128, 64, 0, 2, None) == 1       # no scales
    assert g(A, A, A, A + 4, 256, None, A, 4, 64, 128, 64, 0, 2, None) == 2      # misaligned scales
    assert g(A, A, A, A, 100, None, A, 4, 64, 128, 64, 0, 2, None) == 3          # group not a power of two
    assert g(A, A, A, A, 256, None, A, 4, 64, 128, 64, 0, 0, None) == 5          # f32
    b = bnb4.bnb4_gemm_backward_dq
    assert b(A, A, A, A, 256, A, 4, 100, 128, 64, 0, 2, None) == 4               # N % 8
