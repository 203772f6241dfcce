"""The 4-bit matmuls in fp32 (x, bias and y in float32) against the float64 oracle.

What the fp32 path computes: y_j = sum_k x_k * w_jk (+ b_j), where w_jk =
RN32(code * absmax) is exactly the oracle's dequantized fp32 weight, each
product and sum an fp32 FMA / add ("Feat/mps gemm 4bit bf16", Performance:
gemv_4bit across fp16, bf16 and fp32).  The oracle evaluates the same sum in
float64, so the only difference is fp32 rounding of the sum.

Tolerances, derived from that arithmetic (u = 2^-24):
  * per element, the classical bound for a sum of K products plus a bias
    evaluated in any order: |y_gpu - y_ref| <= gamma_{K+2} (sum_k |x_k w_jk|
    + |b_j|), gamma_n = n u / (1 - n u);
  * over the tensor, rounding errors that do not correlate grow like a random
    walk, sqrt(K) u relative; the relative L2 bound is eight times that.
Both are far tighter than the 5e-3 of the 16-bit paths: a weight rounded to
bf16 or tf32 anywhere would fail them.
"""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_b200 as bnb4
import oracle
import synthetic

from gpu_util import rel_l2, to_dev, to_host

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def gamma(n):
    return n * U / (1 - n * U)


class Weight:
    def __init__(self, N, K, B=64, q="nf4", seed=0, sigma=0.02):
        self.N, self.K, self.B, self.q = N, K, B, q
        w = synthetic.weight(N, K, seed, sigma).numpy().reshape(-1)
        self.packed, self.absmax = oracle.quantize(w, "f32", B, q)
        self.dp = torch.from_numpy(self.packed).cuda()
        self.da = torch.from_numpy(self.absmax).cuda()
        # the exact fp32 dequantized weight, for the per-element bound
        self.wdeq = oracle.dequantize(self.packed, self.absmax, N * K, B, q, "f32").reshape(N, K)


def check(got, ref, absdot, K):
    """got, ref: [.., n] arrays; absdot: the same shape, sum |x w| (+ |b|)."""
    got = np.asarray(got, np.float64)
    bound = gamma(K + 2) * absdot
    worst = np.max(np.abs(got - ref) - bound)
    assert worst <= 0.0, ("per-element bound exceeded by", worst)
    err = rel_l2(got, ref)
    assert err <= 8 * np.sqrt(K) * U, err


def forward_case(M, N, K, B, q, with_bias, seed):
    Wt = Weight(N, K, B, q, seed=seed)
    X = synthetic.activations(M, K, seed=seed + 1, dtype="f32").numpy()
    b = synthetic.bias(N, seed=seed + 2, dtype="f32").numpy() if with_bias else None
    Xd = to_dev(X.reshape(-1), "f32").view(M, K)
    bd = None if b is None else to_dev(b, "f32")
    if M == 1:
        Y = to_host(bnb4.gemv_4bit(Xd.view(-1), Wt.dp, Wt.da, N, K, bd, B, q)).reshape(1, N)
    else:
        Y = to_host(bnb4.gemm_4bit(Xd, Wt.dp, Wt.da, N, bd, B, q)).reshape(M, N)
    ref = oracle.matmul(X.reshape(-1), "f32", Wt.packed, Wt.absmax, b, M, N, K, B, q).reshape(M, N)
    absdot = np.abs(X.astype(np.float64)) @ np.abs(Wt.wdeq.astype(np.float64)).T
    if b is not None:
        absdot = absdot + np.abs(b.astype(np.float64))[None, :]
    check(Y, ref, absdot, K)


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("N,K,B", [(96, 4096, 64), (33, 512, 128), (70, 4672, 64), (64, 2048, 2048),
                                   (17, 128, 64), (40, 8192, 4096), (5, 64, 64), (300, 1024, 256)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemv_f32(q, N, K, B, with_bias):
    forward_case(1, N, K, B, q, with_bias, seed=N + K)


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("M", [2, 3, 16, 17, 64, 100])
@pytest.mark.parametrize("N,K,B", [(96, 512, 64), (200, 1280, 128), (64, 4672, 64), (33, 256, 256)])
def test_gemm_f32(q, M, N, K, B):
    forward_case(M, N, K, B, q, with_bias=M % 2 == 1, seed=M + N)


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("M,N,K,B", [(1, 96, 128, 64), (5, 100, 256, 64), (70, 200, 1280, 128),
                                     (64, 64, 512, 512), (17, 1000, 192, 64)])
def test_gemm_backward_f32(q, M, N, K, B):
    """Includes reductions (N) that are not a multiple of 8 or of the 64-wide step."""
    Wt = Weight(N, K, B, q, seed=N)
    dY = synthetic.grad_output(M, N, seed=3, dtype="f32").numpy()
    dX = to_host(bnb4.gemm_4bit_backward(to_dev(dY.reshape(-1), "f32").view(M, N), Wt.dp, Wt.da, K, B, q))
    ref = oracle.matmul_backward(dY.reshape(-1), "f32", Wt.packed, Wt.absmax, M, N, K, B, q).reshape(M, K)
    absdot = np.abs(dY.astype(np.float64)) @ np.abs(Wt.wdeq.astype(np.float64))
    check(dX.reshape(M, K), ref, absdot, N)


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096)])
def test_gemv_f32_decode_shapes_sampled(K, N):
    """Llama-3-8B-shaped decode projections in fp32, NF4 B=64, with bias: sampled rows."""
    Wt = Weight(N, K, 64, "nf4", seed=0)
    x = synthetic.activations(1, K, seed=1, dtype="f32").numpy().reshape(-1)
    b = synthetic.bias(N, seed=2, dtype="f32").numpy()
    y = to_host(bnb4.gemv_4bit(to_dev(x, "f32"), Wt.dp, Wt.da, N, K, to_dev(b, "f32"), 64, "nf4"))
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(K).integers(0, N, 254)]))
    ref = oracle.matmul_entries(x, "f32", Wt.packed, Wt.absmax, b, 1, N, K, 64, "nf4",
                                np.zeros(rows.size, np.int64), rows)
    absdot = np.abs(Wt.wdeq[rows].astype(np.float64)) @ np.abs(x.astype(np.float64)) + np.abs(b[rows])
    check(y[rows], ref, absdot, K)


@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_gemm_f32_small_m_70b_shapes_sampled(K, N):
    """Llama-3-70B-shaped small-M projections in fp32 (NF4 B=64, bias), in the
    launch the bench times: M = 4, 8 and 16, sampled output columns."""
    w = synthetic.weight(N, K, 0, 0.015).numpy().reshape(-1)
    packed, absmax = oracle.quantize(w, "f32", 64, "nf4")
    del w
    dp, da = torch.from_numpy(packed).cuda(), torch.from_numpy(absmax).cuda()
    b = synthetic.bias(N, seed=2, dtype="f32").numpy()
    cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(N).integers(0, N, 126)]))
    # the sampled rows of the exact fp32 weight, for the per-element bound
    rb = K // 2
    wsel = np.stack([oracle.dequantize(packed[c * rb:(c + 1) * rb], absmax[c * (K // 64):(c + 1) * (K // 64)],
                                       K, 64, "nf4", "f32") for c in cols]).astype(np.float64)
    for M in (4, 8, 16):
        X = synthetic.activations(M, K, seed=M, dtype="f32").numpy()
        Y = to_host(bnb4.gemm_4bit(to_dev(X.reshape(-1), "f32").view(M, K), dp, da, N,
                                   to_dev(b, "f32"), 64, "nf4")).reshape(M, N)
        ms = np.repeat(np.arange(M), cols.size)
        ns = np.tile(cols, M)
        ref = oracle.matmul_entries(X.reshape(-1), "f32", packed, absmax, b, M, N, K, 64, "nf4", ms, ns)
        absdot = (np.abs(X.astype(np.float64)) @ np.abs(wsel).T + np.abs(b[cols])[None, :]).reshape(-1)
        check(Y[ms, ns], ref, absdot, K)
