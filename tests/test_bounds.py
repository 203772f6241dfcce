"""The per-element error bound of the 16-bit matmul tests, checked on the CPU.

A numpy restatement of what the 16-bit kernels compute (the weight rounded
once to the compute dtype, fp32 products and sums, one rounding of the
output) must lie inside the bound; the same arithmetic with one planted
mistake (one block's absmax scaled by 1.5) must fall outside it, although it still
passes the relative L2 bar over the whole output.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic

from gpu_util import MATMUL_TOL, as_f64, elementwise_excess, rel_l2


def _round16(a32, dt):
    t = torch.from_numpy(np.ascontiguousarray(a32, np.float32))
    return t.to(torch.bfloat16 if dt == "bf16" else torch.float16).to(torch.float32).numpy()


def _emulate(Xs, dt, packed, absmax, M, N, K, B, q, kernel_style):
    """fp32 emulation of the 16-bit matmul: weight RN_dt(code) * absmax (M <= 16
    kernels) or RN_dt(code * absmax) (tcgen05 kernel), fp32 sum, output RN_dt."""
    x = as_f64(Xs, dt).astype(np.float32).reshape(M, K)
    codes = np.asarray(oracle.code_table(q), np.float32)
    idx = np.empty(N * K, np.uint8)
    idx[0::2] = packed >> 4
    idx[1::2] = packed & 15
    a = np.repeat(absmax, B)[: N * K].astype(np.float32)
    if kernel_style == "small":
        w = (_round16(codes[idx], dt) * a).astype(np.float32)
    else:
        w = _round16((codes[idx] * a).astype(np.float32), dt)
    y32 = (x @ w.reshape(N, K).T).astype(np.float32)
    return _round16(y32, dt).astype(np.float64)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("style", ["small", "tc"])
def test_restatement_inside_and_planted_mistake_outside(dt, style):
    M, N, K, B, q = 12, 8192, 256, 64, "nf4"
    w = synthetic.weight(N, K, 0).numpy().reshape(-1)
    packed, absmax = oracle.quantize(w, "f32", B, q)
    Xs = synthetic.storage_numpy(synthetic.activations(M, K, seed=1, dtype=dt)).reshape(-1)
    ref = oracle.matmul(Xs, dt, packed, absmax, None, M, N, K, B, q)
    wdeq = oracle.dequantize(packed, absmax, N * K, B, q, "f32").astype(np.float64).reshape(N, K)
    absdot = np.abs(as_f64(Xs, dt).reshape(M, K)) @ np.abs(wdeq).T
    good = _emulate(Xs, dt, packed, absmax, M, N, K, B, q, style)
    assert rel_l2(good, ref) <= MATMUL_TOL
    assert elementwise_excess(good, ref, absdot, dt, K) <= 0
    bad_absmax = absmax.copy()
    bad_absmax[7 * (K // B) + 2] *= 1.5      # row 7, its third block
    bad = _emulate(Xs, dt, packed, bad_absmax, M, N, K, B, q, style)
    assert rel_l2(bad, ref) <= MATMUL_TOL    # the global bar does not see it
    assert elementwise_excess(bad, ref, absdot, dt, K) > 0
