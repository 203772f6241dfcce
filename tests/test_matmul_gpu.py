"""gemv_4bit / gemm_4bit / gemm_4bit_backward on the GPU against the float64 oracle.

Bar: relative L2 error <= 5e-3 (bf16/fp16 out, fp32 accumulate) against the
float64 product of the oracle's dequantized (fp32) weights.
"""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_b200 as bnb4
import oracle
import synthetic

from gpu_util import MATMUL_TOL, as_f64, elementwise_excess, rel_l2, to_dev, to_host

pytestmark = pytest.mark.gpu


class Weight:
    """A seeded fp32 weight [N, K] quantized by the oracle (the GPU path gets the same bytes)."""

    def __init__(self, N, K, B=64, q="nf4", seed=0, sigma=0.02):
        self.N, self.K, self.B, self.q = N, K, B, q
        w = synthetic.weight(N, K, seed, sigma).numpy().reshape(-1)
        self.packed, self.absmax = oracle.quantize(w, "f32", B, q)
        self.dp = torch.from_numpy(self.packed).cuda()
        self.da = torch.from_numpy(self.absmax).cuda()
        self._absw = None

    def absw(self):
        """|dequantized fp32 weight| [N, K] in float64 (for the per-element bounds)."""
        if self._absw is None:
            w = oracle.dequantize(self.packed, self.absmax, self.N * self.K, self.B, self.q, "f32")
            self._absw = np.abs(w.astype(np.float64)).reshape(self.N, self.K)
        return self._absw

    def absw_rows(self, rows):
        """|dequantized fp32 weight| of the given rows only, [len(rows), K] float64."""
        hb, nb = self.K // 2, self.K // self.B
        p = np.concatenate([self.packed[r * hb:(r + 1) * hb] for r in rows])
        a = np.concatenate([self.absmax[r * nb:(r + 1) * nb] for r in rows])
        w = oracle.dequantize(p, a, len(rows) * self.K, self.B, self.q, "f32")
        return np.abs(w.astype(np.float64)).reshape(len(rows), self.K)


def _absdot(Xs, dt, absw_rows, bias_s=None):
    """sum_k |x_mk w_jk| (+ |b_j|) for every (m, j) of X [M, K] and the given weight rows."""
    K = absw_rows.shape[1]
    ax = np.abs(as_f64(Xs, dt)).reshape(-1, K)
    d = ax @ absw_rows.T
    if bias_s is not None:
        d = d + np.abs(as_f64(bias_s, dt))[None, :]
    return d


def _ref_forward(Wt, Xs, dt, bias_s, rows=None):
    M = Xs.size // Wt.K
    if rows is None:
        return oracle.matmul(Xs, dt, Wt.packed, Wt.absmax, bias_s, M, Wt.N, Wt.K, Wt.B, Wt.q)
    ms = np.repeat(np.arange(M), rows.size)
    js = np.tile(rows, M)
    v = oracle.matmul_entries(Xs, dt, Wt.packed, Wt.absmax, bias_s, M, Wt.N, Wt.K, Wt.B, Wt.q,
                              ms, js)
    return v.reshape(M, rows.size)


# ----------------------------------------------------------------------- gemv

@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("N,K,B", [(96, 4096, 64), (33, 512, 128), (70, 4672, 64),
                                   (64, 2048, 2048), (200, 1024, 1024), (17, 128, 64),
                                   (40, 8192, 4096)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemv_small_shapes(q, dt, N, K, B, with_bias):
    Wt = Weight(N, K, B, q, seed=N + K)
    xs = synthetic.storage_numpy(synthetic.activations(1, K, seed=1, dtype=dt)).reshape(-1)
    bs = synthetic.storage_numpy(synthetic.bias(N, seed=2, dtype=dt)) if with_bias else None
    y = bnb4.gemv_4bit(to_dev(xs, dt), Wt.dp, Wt.da, N, K, None if bs is None else to_dev(bs, dt),
                       B, q)
    ref = _ref_forward(Wt, xs, dt, bs)[0]
    got = as_f64(to_host(y), dt)
    err = rel_l2(got, ref)
    assert err <= MATMUL_TOL, err
    assert elementwise_excess(got, ref, _absdot(xs, dt, Wt.absw(), bs)[0], dt, K) <= 0


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemv_llama_decode_shapes_sampled(K, N, with_bias):
    """Llama-3-8B-shaped decode projections, NF4 blocksize 64, bf16: sampled rows."""
    Wt = Weight(N, K, 64, "nf4", seed=0, sigma=0.02)
    xs = synthetic.storage_numpy(synthetic.activations(1, K, seed=1)).reshape(-1)
    bs = synthetic.storage_numpy(synthetic.bias(N, seed=2)) if with_bias else None
    y = to_host(bnb4.gemv_4bit(to_dev(xs, "bf16"), Wt.dp, Wt.da, N, K,
                               None if bs is None else to_dev(bs, "bf16"), 64, "nf4"))
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(K + N).integers(0, N, 254)]))
    ref = _ref_forward(Wt, xs, "bf16", bs, rows)[0]
    got = as_f64(y, "bf16")[rows]
    err = rel_l2(got, ref)
    assert err <= MATMUL_TOL, err
    ad = _absdot(xs, "bf16", Wt.absw_rows(rows))[0] + (0 if bs is None else np.abs(as_f64(bs, "bf16"))[rows])
    assert elementwise_excess(got, ref, ad, "bf16", K) <= 0


# -------------------------------------------------------------- small-M gemm

@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 9, 16])
@pytest.mark.parametrize("N,K,B", [(96, 2048, 64), (45, 1600, 64), (64, 4096, 256),
                                   (33, 1024, 1024)])
def test_gemm_small_m(q, dt, M, N, K, B):
    Wt = Weight(N, K, B, q, seed=M + N)
    Xs = synthetic.storage_numpy(synthetic.activations(M, K, seed=1, dtype=dt)).reshape(-1)
    bs = synthetic.storage_numpy(synthetic.bias(N, seed=2, dtype=dt)) if M % 2 else None
    Y = bnb4.gemm_4bit(to_dev(Xs, dt).view(M, K), Wt.dp, Wt.da, N,
                       None if bs is None else to_dev(bs, dt), B, q)
    ref = _ref_forward(Wt, Xs, dt, bs)
    got = as_f64(to_host(Y), dt).reshape(M, N)
    err = rel_l2(got, ref)
    assert err <= MATMUL_TOL, err
    assert elementwise_excess(got, ref, _absdot(Xs, dt, Wt.absw(), bs), dt, K) <= 0


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_gemm_small_m_70b_shapes_sampled(q, dt, K, N):
    """70B-shaped projections, M in {1,2,4,8,16}, sigma 0.015: sampled rows."""
    Wt = Weight(N, K, 64, q, seed=0, sigma=0.015)
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(K).integers(0, N, 62)]))
    absw_r = Wt.absw_rows(rows)
    for M in (1, 2, 4, 8, 16):
        Xs = synthetic.storage_numpy(synthetic.activations(M, K, seed=1, dtype=dt)).reshape(-1)
        Y = to_host(bnb4.gemm_4bit(to_dev(Xs, dt).view(M, K), Wt.dp, Wt.da, N, None, 64, q))
        ref = _ref_forward(Wt, Xs, dt, None, rows)
        got = as_f64(Y, dt).reshape(M, N)[:, rows]
        err = rel_l2(got, ref)
        assert err <= MATMUL_TOL, (M, err)
        assert elementwise_excess(got, ref, _absdot(Xs, dt, absw_r), dt, K) <= 0, M


# ---------------------------------------------- large-M gemm and backward (tcgen05)

def _ref_backward(Wt, dYs, dt, M, entries=None):
    if entries is None:
        return oracle.matmul_backward(dYs, dt, Wt.packed, Wt.absmax, M, Wt.N, Wt.K, Wt.B, Wt.q)
    ms, ks = entries
    return oracle.matmul_backward_entries(dYs, dt, Wt.packed, Wt.absmax, M, Wt.N, Wt.K, Wt.B,
                                          Wt.q, ms, ks)


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("M,N,K,B", [(17, 256, 256, 64), (100, 320, 512, 64), (256, 512, 1024, 128),
                                     (300, 96, 256, 256), (257, 264, 704, 64), (300, 256, 4096, 64),
                                     (300, 33152, 256, 64), (300, 33152, 192, 64)])
def test_gemm_large_m(q, dt, M, N, K, B):
    """Includes a reduction split over a cluster (K=4096, two tiles), a width
    (N = 148 * 224) where 224-column tiles fill the SMs, and absmax rows whose
    pitch (K / B scales) is not a multiple of four (K = 704, 192 at B = 64;
    K = 256 at B = 256)."""
    Wt = Weight(N, K, B, q, seed=M)
    Xs = synthetic.storage_numpy(synthetic.activations(M, K, seed=1, dtype=dt)).reshape(-1)
    bs = synthetic.storage_numpy(synthetic.bias(N, seed=2, dtype=dt)) if M % 2 == 0 else None
    Y = bnb4.gemm_4bit(to_dev(Xs, dt).view(M, K), Wt.dp, Wt.da, N,
                       None if bs is None else to_dev(bs, dt), B, q)
    ref = _ref_forward(Wt, Xs, dt, bs)
    got = as_f64(to_host(Y), dt).reshape(M, N)
    err = rel_l2(got, ref)
    assert err <= MATMUL_TOL, err
    assert elementwise_excess(got, ref, _absdot(Xs, dt, Wt.absw(), bs), dt, K) <= 0


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("M,N,K,B", [(1, 256, 256, 64), (17, 256, 512, 64), (256, 200, 256, 64),
                                     (300, 320, 768, 256), (64, 1024, 1280, 128),
                                     (64, 8192, 256, 64), (300, 4096, 512, 128),
                                     (130, 264, 2048, 128), (96, 520, 3072, 512)])
def test_gemm_backward(q, dt, M, N, K, B):
    """Includes reductions long enough to be split over a thread-block cluster,
    ragged reductions (N = 200, 264, 520), blocks of 128 scales shared by two
    64-column groups of a tile, and absmax pitches that are not a multiple of
    four scales (K / B = 3, 10, 6)."""
    Wt = Weight(N, K, B, q, seed=N)
    dYs = synthetic.storage_numpy(synthetic.grad_output(M, N, seed=3, dtype=dt)).reshape(-1)
    dX = bnb4.gemm_4bit_backward(to_dev(dYs, dt).view(M, N), Wt.dp, Wt.da, K, B, q)
    ref = _ref_backward(Wt, dYs, dt, M)
    got = as_f64(to_host(dX), dt).reshape(M, K)
    err = rel_l2(got, ref)
    assert err <= MATMUL_TOL, err
    ad = np.abs(as_f64(dYs, dt)).reshape(M, N) @ Wt.absw()
    assert elementwise_excess(got, ref, ad, dt, N) <= 0


@pytest.mark.parametrize("M", [512, 2048])
def test_prefill_and_backward_full_size_sampled(M):
    """M in {512, 2048}, K=4096, N=14336, NF4 B=64, bf16: sampled outputs of both passes."""
    K, N = 4096, 14336
    Wt = Weight(N, K, 64, "nf4", seed=0, sigma=0.02)
    rng = np.random.default_rng(M)
    Xs = synthetic.storage_numpy(synthetic.activations(M, K, seed=1)).reshape(-1)
    Y = as_f64(to_host(bnb4.gemm_4bit(to_dev(Xs, "bf16").view(M, K), Wt.dp, Wt.da, N)),
               "bf16").reshape(M, N)
    ms = np.concatenate([[0, M - 1, M - 1], rng.integers(0, M, 509)])
    js = np.concatenate([[0, N - 1, 0], rng.integers(0, N, 509)])
    ref = oracle.matmul_entries(Xs, "bf16", Wt.packed, Wt.absmax, None, M, N, K, 64, "nf4", ms, js)
    err = rel_l2(Y[ms, js], ref)
    assert err <= MATMUL_TOL, ("forward", err)
    ax = np.abs(as_f64(Xs, "bf16")).reshape(M, K)
    aw = Wt.absw()
    assert elementwise_excess(Y[ms, js], ref, (ax[ms] * aw[js]).sum(1), "bf16", K) <= 0, "forward"
    dYs = synthetic.storage_numpy(synthetic.grad_output(M, N, seed=3)).reshape(-1)
    dX = as_f64(to_host(bnb4.gemm_4bit_backward(to_dev(dYs, "bf16").view(M, N), Wt.dp, Wt.da, K)),
                "bf16").reshape(M, K)
    ks = np.concatenate([[0, K - 1, 0], rng.integers(0, K, 253)])
    ms2 = ms[:ks.size]
    refb = _ref_backward(Wt, dYs, "bf16", M, (ms2, ks))
    err = rel_l2(dX[ms2, ks], refb)
    assert err <= MATMUL_TOL, ("backward", err)
    ady = np.abs(as_f64(dYs, "bf16")).reshape(M, N)
    assert elementwise_excess(dX[ms2, ks], refb, (ady[ms2] * aw[:, ks].T).sum(1), "bf16", N) <= 0, "backward"
