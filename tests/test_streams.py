"""Stream ordering: every call runs on the stream it is given, after the work
already queued there, with no host synchronisation.

The pages' race test ("Feat/mps gemm 4bit bf16", Correctness) failed 30 of 30
iterations once the synchronisation before dispatch was removed: kernels read
inputs that a producer had not yet written.  Here the inputs are written on a
side stream by a copy queued behind a bounded spin (torch.cuda._sleep, a fixed
cycle count), then consumed by the library on that stream (or on another stream
that waits on an event); the host never synchronises in between.  A call that
ran on the wrong stream, or early, would read the stale contents (NaN or
another iteration's data) and fail the bit-exact comparison with the oracle.
"""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_b200 as bnb4
import oracle
import synthetic

from gpu_util import MATMUL_TOL, as_f64, rel_l2, to_dev, to_host

pytestmark = pytest.mark.gpu

SPIN = 20_000_000   # GPU cycles, about 10 ms at B200 clocks: long enough for every launch to queue


def _pinned(t):
    return t.contiguous().pin_memory()


def test_quantize_gemv_dequantize_behind_a_slow_producer_30_iterations():
    n, B = (1 << 16) + 77, 64
    N, K = 256, 1024
    w = synthetic.weight(N, K, 0).numpy().reshape(-1)
    wp, wa = oracle.quantize(w, "f32", B, "nf4")
    dp, da = torch.from_numpy(wp).cuda(), torch.from_numpy(wa).cuda()
    side = torch.cuda.Stream()
    x_dev = torch.full((n,), float("nan"), dtype=torch.bfloat16, device="cuda")
    v_dev = torch.full((K,), float("nan"), dtype=torch.bfloat16, device="cuda")
    packed = torch.empty((n + 1) // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty((n + B - 1) // B, dtype=torch.float32, device="cuda")
    deq = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(N, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    for it in range(30):
        x = synthetic.roundtrip_tensor(n, it, "bf16")
        v = synthetic.activations(1, K, seed=100 + it).reshape(-1)
        hx, hv = _pinned(x), _pinned(v)
        with torch.cuda.stream(side):
            torch.cuda._sleep(SPIN)
            x_dev.copy_(hx, non_blocking=True)
            v_dev.copy_(hv, non_blocking=True)
        # the library gets the side stream explicitly; torch's current stream is the default one
        bnb4.quantize_4bit_into(x_dev, packed, absmax, B, "nf4", stream=side)
        bnb4.dequantize_4bit(packed, absmax, n, B, "nf4", out=deq, stream=side)
        bnb4.gemv_4bit(v_dev, dp, da, N, K, None, B, "nf4", out=y, stream=side)
        side.synchronize()
        op, oa = oracle.quantize(synthetic.storage_numpy(x), "bf16", B, "nf4")
        assert np.array_equal(to_host(packed), op) and np.array_equal(to_host(absmax), oa), it
        assert np.array_equal(to_host(deq), oracle.dequantize(op, oa, n, B, "nf4", "bf16")), it
        vs = synthetic.storage_numpy(v)
        ref = oracle.matmul(vs, "bf16", wp, wa, None, 1, N, K, B, "nf4")[0]
        assert rel_l2(as_f64(to_host(y), "bf16"), ref) <= MATMUL_TOL, it
        # the next iteration's producer overwrites the inputs: poison them first
        with torch.cuda.stream(side):
            x_dev.fill_(float("nan"))
            v_dev.fill_(float("nan"))


def test_consumer_stream_waits_on_a_producer_event():
    """Producer on one stream, library calls on another stream that waits on an
    event recorded after the producer's write."""
    n, B = 1 << 18, 128
    prod, cons = torch.cuda.Stream(), torch.cuda.Stream()
    x = synthetic.roundtrip_tensor(n, 7, "f16")
    x_dev = torch.full((n,), float("nan"), dtype=torch.float16, device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(prod):
        torch.cuda._sleep(SPIN)
        x_dev.copy_(_pinned(x), non_blocking=True)
        done = torch.cuda.Event()
        done.record(prod)
    cons.wait_event(done)
    packed, absmax = bnb4.quantize_4bit(x_dev, B, "fp4", stream=cons)
    cons.synchronize()
    op, oa = oracle.quantize(synthetic.storage_numpy(x), "f16", B, "fp4")
    assert np.array_equal(to_host(packed), op) and np.array_equal(to_host(absmax), oa)


def test_two_streams_on_disjoint_buffers_at_once():
    """Two independent pipelines (quantize, 8-bit statistics, small-M gemm) on
    two streams, each behind its own spin, overlapping on the GPU."""
    B = 64
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    cases = []
    for i, (N, K, M, dt) in enumerate([(192, 2048, 8, "bf16"), (160, 1024, 4, "f16")]):
        w = synthetic.weight(N, K, 10 + i).numpy().reshape(-1)
        Xs = synthetic.storage_numpy(synthetic.activations(M, K, seed=20 + i, dtype=dt)).reshape(-1)
        cases.append((N, K, M, dt, w, Xs))
    torch.cuda.synchronize()
    outs = []
    for (N, K, M, dt, w, Xs), s in zip(cases, streams):
        wd = torch.full((N * K,), float("nan"), device="cuda")
        Xd = torch.full((M * K,), float("nan"), dtype=synthetic.TORCH_DTYPES[dt], device="cuda")
        s.wait_stream(torch.cuda.current_stream())   # the NaN fills above come first
        with torch.cuda.stream(s):
            torch.cuda._sleep(SPIN)
            wd.copy_(_pinned(torch.from_numpy(w)), non_blocking=True)
            Xd.copy_(_pinned(to_dev(Xs, dt).cpu()), non_blocking=True)
        p, a = bnb4.quantize_4bit(wd, B, "nf4", stream=s)
        q8, s8 = bnb4.double_quant(a, 256, stream=s)
        Y = bnb4.gemm_4bit_dq(Xd.view(M, K), p, q8, s8, N, None, B, "nf4", 256, stream=s)
        outs.append((p, a, q8, s8, Y))
    for s in streams:
        s.synchronize()
    for (N, K, M, dt, w, Xs), (p, a, q8, s8, Y) in zip(cases, outs):
        op, oa = oracle.quantize(w, "f32", B, "nf4")
        assert np.array_equal(to_host(p), op) and np.array_equal(to_host(a), oa)
        oq, osc = oracle.double_quant(oa, 256)
        assert np.array_equal(to_host(q8), oq) and np.array_equal(to_host(s8), osc)
        back = oracle.dequant_absmax(oq, osc, 256)
        ref = oracle.matmul(Xs, dt, op, back, None, M, N, K, B, "nf4")
        assert rel_l2(as_f64(to_host(Y), dt).reshape(M, N), ref) <= MATMUL_TOL


def test_chained_gemvs_read_the_previous_output():
    """Twenty gemv launches back to back, each reading the one before it as its
    x (4096 -> 1024 -> 4096 ...), no host synchronisation.  The gemv may start
    before the previous kernel ends (programmatic dependent launch); it must
    still read that kernel's finished output.  Each step is compared with the
    oracle applied to the previous step's GPU output."""
    K1, N1 = 4096, 1024
    B = 64
    ws = []
    for (N, K, seed) in ((N1, K1, 31), (K1, N1, 32)):
        w = synthetic.weight(N, K, seed, sigma=1.0 / np.sqrt(K)).numpy().reshape(-1)
        p, a = oracle.quantize(w, "f32", B, "nf4")
        ws.append((N, K, p, a, torch.from_numpy(p).cuda(), torch.from_numpy(a).cuda()))
    v0 = synthetic.activations(1, K1, seed=33).reshape(-1).cuda()
    outs = []
    x = v0
    torch.cuda.synchronize()
    torch.cuda._sleep(SPIN)                  # the chain queues up behind a long kernel
    for i in range(20):
        N, K, p, a, dp, da = ws[i % 2]
        y = torch.empty(N, dtype=torch.bfloat16, device="cuda")
        bnb4.gemv_4bit(x, dp, da, N, K, None, B, "nf4", out=y)
        outs.append(y)
        x = y
    torch.cuda.synchronize()
    prev = synthetic.storage_numpy(v0.cpu())
    for i, y in enumerate(outs):
        N, K, p, a, _, _ = ws[i % 2]
        ref = oracle.matmul(prev, "bf16", p, a, None, 1, N, K, B, "nf4")[0]
        got = to_host(y)
        assert rel_l2(as_f64(got, "bf16"), ref) <= MATMUL_TOL, i
        prev = got
