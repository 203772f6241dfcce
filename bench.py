"""Benchmark of the 4-bit blockwise weight path on B200.

One step = one pass of the whole hot path over one batch of seeded synthetic
input:
  1. quantize_4bit     x[2^28] bf16 ~N(0,1) + 1% x20 outliers -> NF4, blocksize 64
  2. gemv_4bit + bias  Llama-3-8B decode projections (K,N) = (4096,4096),
                       (4096,1024), (4096,14336), (14336,4096); NF4 B=64, bf16
  3. gemm_4bit M=16    70B-shaped (K,N) = (8192,28672), (28672,8192)
  4. gemm_4bit M=512   prefill, K=4096, N=14336
  5. gemm_4bit_backward M=512 (grad_input = grad_out @ dequant(W))
  6. dequantize_4bit   the step-1 result back to bf16 (after 2-5 have evicted it from L2)
Throughput (GB/s) = algorithmic bytes of the step / step time; the step's
working set (~1.6 GB) is far larger than L2, so every kernel reads cold data.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (the plain C restatement of the
method) on a bounded sample of the same workload.  Under torchrun every rank
runs its own independent batch (weak scaling, no collective on the data
path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_ELEMS = 1 << 28
BLOCK = 64
CLOCK_MHZ_NOMINAL = 1965   # B200 maximum SM clock (the fp32 FMA rate is computed at it)
GEMV_SHAPES = [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)]
SMALLM_SHAPES = [(8192, 28672), (28672, 8192)]
SMALLM_M = 16
PREFILL = (512, 4096, 14336)  # M, K, N
METRIC = "gemv_4bit NF4 decode GB/s & % of HBM roofline; quantize_4bit GB/s"
WORKLOAD = ("full 4-bit hot path per step: quantize 2^28 bf16 (NF4, B=64) + gemv+bias on 4 "
            "Llama-3-8B decode shapes + M=16 gemm on 2 70B shapes + M=512 prefill gemm "
            "(K=4096, N=14336) and its backward + dequantize 2^28")


def wbytes(N, K):
    return N * K // 2 + N * K // BLOCK * 4


def step_ops():
    """(name, algorithmic bytes, flops) for each launch of one step, in order."""
    ops = [("quantize_4bit", N_ELEMS * 2 + N_ELEMS // 2 + N_ELEMS // BLOCK * 4, 0)]
    for K, N in GEMV_SHAPES:
        ops.append((f"gemv_4bit_{K}x{N}", wbytes(N, K) + 2 * K + 2 * N + 2 * N, 2 * N * K))
    for K, N in SMALLM_SHAPES:
        M = SMALLM_M
        ops.append((f"gemm_4bit_M{M}_{K}x{N}", wbytes(N, K) + 2 * M * K + 2 * M * N, 2 * M * N * K))
    M, K, N = PREFILL
    ops.append((f"gemm_4bit_M{M}_{K}x{N}", wbytes(N, K) + 2 * M * K + 2 * M * N, 2 * M * N * K))
    ops.append((f"gemm_4bit_backward_M{M}_{K}x{N}", wbytes(N, K) + 2 * M * N + 2 * M * K,
                2 * M * N * K))
    ops.append(("dequantize_4bit", N_ELEMS // 2 + N_ELEMS // BLOCK * 4 + N_ELEMS * 2, 0))
    return ops


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), \
            "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_src_hash(fname):
    with open(os.path.join(ROOT, "bit_blockwise_weight_b200", "csrc", fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(op_name):
    """DRAM bytes per launch recorded by an ncu capture under profiles/, or None when
    the kernel source has changed since (the summary records the source hash)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(op_name)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("src_sha256_16") != kernel_src_hash(rec["src"]):
        return None
    return rec["dram_bytes_per_launch"]


SRC_OF = {"quantize_4bit": "quant.cu", "dequantize_4bit": "quant.cu"}


def src_of(op):
    if op in SRC_OF:
        return SRC_OF[op]
    if op.startswith("gemv"):
        return "gemv.cu"
    if "backward" in op or "_M512_" in op:
        return "gemm_tc.cu"
    return "gemm_small.cu"


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML every few ms while the
    timed region runs; stop() returns None when NVML cannot be used."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, dev):
        self.dev = dev
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.stop_ev = threading.Event()
        self.t = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(self.dev)
            # NVML wants the bus id as text ("DDDDDDDD:BB:DD.0"); torch gives integers
            bus = "%08X:%02X:%02X.0" % (int(props.pci_domain_id), int(props.pci_bus_id),
                                        int(props.pci_device_id))
            try:
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except pynvml.NVMLError:
                h = pynvml.nvmlDeviceGetHandleByIndex(int(self.dev.index))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")

            def run():
                while not self.stop_ev.is_set():
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    r = get_reasons(h)
                    for nm, bit in self.REASONS.items():
                        if r & bit:
                            self.reasons.add(nm)
                    time.sleep(0.002)
            self.t = threading.Thread(target=run, daemon=True)
            self.t.start()
            # the first sample is taken before the timed region starts
            t_end = time.time() + 0.2
            while not self.samples and time.time() < t_end:
                time.sleep(0.001)
        except Exception:
            self.t = None

    def stop(self):
        if self.t is None:
            return None
        self.stop_ev.set()
        self.t.join(timeout=2)
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------ across the ranks

def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time.  Every rank calls this at the same point, in
    the same order (it is a collective when world > 1)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job rate per second: the units all ranks processed (each rank runs its
    own batch of the same size) over the slowest rank's time for `steps` steps."""
    return units_per_rank_step * steps * world / (ms / 1e3)


def roofline_and_parts(ops, per_op_ms, hbm, tc_burst, tc_sust, peak_kind, traffic=None):
    """The roofline object for the op with the largest time share (HBM GB/s, or
    TFLOP/s for the tensor-core matmuls) and the per-op breakdown.
    ops: (name, algorithmic bytes, flops) per launch; per_op_ms: mean durations.
    A tensor-core op is judged against the burst bf16 peak (its launches are tens
    of microseconds inside a sub-millisecond step, not a seconds-long loop under
    the power cap); the fraction of the sustained peak is reported beside it."""
    traffic = traffic or profiled_traffic
    di = max(range(len(per_op_ms)), key=lambda i: per_op_ms[i])
    name, nbytes, nflops = ops[di]
    if nflops and "_M512_" in name:
        achieved = nflops / (per_op_ms[di] / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tc_burst,
                "unit": "TFLOP/s", "frac": round(achieved / tc_burst, 4),
                "frac_of_sustained": round(achieved / tc_sust, 4),
                "traffic": traffic(name), "kernel": name,
                "peak_kind": f"{peak_kind} burst bf16 (sustained {tc_sust})"}
    else:
        achieved = nbytes / (per_op_ms[di] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": traffic(name),
                "kernel": name, "peak_kind": f"{peak_kind} HBM copy"}
    parts = {}
    total = sum(per_op_ms)
    for (nm, nb, nf), t in zip(ops, per_op_ms):
        e = {"us": round(t * 1e3, 2), "GB/s": round(nb / (t / 1e3) / 1e9, 1),
             "hbm_frac": round(nb / (t / 1e3) / 1e9 / hbm, 4),
             "share": round(t / total, 4)}
        if "_M512_" in nm:
            e["TFLOP/s"] = round(nf / (t / 1e3) / 1e12, 1)
            e["tensor_frac"] = round(nf / (t / 1e3) / 1e12 / tc_burst, 4)
            e["tensor_frac_of_sustained"] = round(nf / (t / 1e3) / 1e12 / tc_sust, 4)
        parts[nm] = e
    return roof, parts


def graph_per_launch(dev, fns, reps=5):
    """Mean device time of one launch, in microseconds: the launches (zero-argument
    callables) captured back to back in one CUDA graph, replayed `reps` times
    between two events on the stream the replays run on, after one untimed
    replay.  The
    callers rotate inputs whose total size exceeds L2, so every launch reads cold
    data."""
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    for f in fns[:2]:
        f()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for f in fns:
            f()
    torch.cuda.synchronize(dev)
    g.replay()
    torch.cuda.synchronize(dev)
    # replay() launches on the current stream: the events go there too
    cur = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(reps):
        g.replay()
    e1.record(cur)
    torch.cuda.synchronize(dev)
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * len(fns))


def copies_for(nbytes, floor_bytes=640 << 20):
    """How many rotating copies of an input of `nbytes` keep the working set of
    one pass above five times L2."""
    return max(2, -(-floor_bytes // max(nbytes, 1)))


def time_configs(dev, hbm, tc_burst, tc_sust):
    """Every workload configuration of the path, each op timed on its own with
    graph_per_launch: quantize/dequantize 2^28 (3 dtypes x NF4/FP4 x 7
    blocksizes), the gemv decode shapes with and without bias (the 4096 x 4096
    one is the gemv NF4 workload), small-M decode on the 70B shapes (M = 1, 2,
    4, 8, 16 x NF4/FP4 x bf16/fp16) and prefill M = 512 / 2048 forward and
    backward."""
    import bit_blockwise_weight_b200 as b
    import synthetic
    d = str(dev)
    out = {}

    def rec(name, us, nbytes, flops=0):
        e = {"us": round(us, 2), "bytes": int(nbytes), "GB/s": round(nbytes / (us / 1e6) / 1e9, 1),
             "hbm_frac": round(nbytes / (us / 1e6) / 1e9 / hbm, 4)}
        if flops:
            tf = flops / (us / 1e6) / 1e12
            e.update({"TFLOP/s": round(tf, 1), "tensor_frac": round(tf / tc_burst, 4),
                      "tensor_frac_of_sustained": round(tf / tc_sust, 4)})
        out[name] = e

    def qweight(N, K, sigma, seed, qt, copies):
        w = synthetic.normal((N * K,), seed, sigma, "f32", device=d)
        p, a = b.quantize_4bit(w, BLOCK, qt)
        del w
        return [p] + [p.clone() for _ in range(copies - 1)], [a] + [a.clone() for _ in range(copies - 1)]

    # quantize / dequantize round trip, 2^28 elements (the input is 0.5-1 GB: each
    # launch reads cold data)
    n = N_ELEMS
    packed = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
    for dt, tdt in (("f32", torch.float32), ("f16", torch.float16), ("bf16", torch.bfloat16)):
        x = synthetic.roundtrip_tensor(n, 0, dt, device=d)
        y = torch.empty(n, dtype=tdt, device=dev)
        s = x.element_size()
        for qt in ("nf4", "fp4"):
            for B in (64, 128, 256, 512, 1024, 2048, 4096):
                nb = n * s + n // 2 + 4 * (n // B)
                a_ = absmax[: n // B]
                us = graph_per_launch(dev, [lambda: b.quantize_4bit_into(x, packed, a_, B, qt)] * 2, reps=3)
                rec(f"quantize_4bit_2p28_{dt}_{qt}_B{B}", us, nb)
                us = graph_per_launch(dev, [lambda: b.dequantize_4bit(packed, a_, n, B, qt, out=y)] * 2, reps=3)
                rec(f"dequantize_4bit_2p28_{dt}_{qt}_B{B}", us, nb)
        del x, y
    del packed, absmax

    # gemv decode shapes (the 4096 x 4096 NF4 one without bias is the gemv NF4 workload)
    for K, N in GEMV_SHAPES:
        nbw = wbytes(N, K)
        C = copies_for(nbw)
        ps, as_ = qweight(N, K, 0.02, 0, "nf4", C)
        xv = synthetic.normal((K,), 1, 1.0, "bf16", device=d)
        bias = synthetic.normal((N,), 2, 1.0, "bf16", device=d)
        y = torch.empty(N, dtype=torch.bfloat16, device=dev)
        for with_bias in (False, True):
            fns = [lambda i=i: b.gemv_4bit(xv, ps[i], as_[i], N, K, bias if with_bias else None, BLOCK, "nf4",
                                           out=y) for i in range(C)]
            us = graph_per_launch(dev, fns)
            rec(f"gemv_4bit_nf4_bf16_{K}x{N}" + ("_bias" if with_bias else ""), us,
                nbw + 2 * K + 2 * N + (2 * N if with_bias else 0), 2 * N * K)
        del ps, as_

    # small-M decode, 70B-shaped (133 MB of weight: two rotating copies)
    for K, N in SMALLM_SHAPES:
        nbw = wbytes(N, K)
        for qt in ("nf4", "fp4"):
            ps, as_ = qweight(N, K, 0.015, 0, qt, 2)
            for dt, tdt in (("bf16", torch.bfloat16), ("f16", torch.float16)):
                for M in (1, 2, 4, 8, 16):
                    X = synthetic.normal((M, K), 1, 1.0, dt, device=d)
                    Y = torch.empty(M, N, dtype=tdt, device=dev)
                    fns = [lambda i=i: b.gemm_4bit(X, ps[i], as_[i], N, None, BLOCK, qt, out=Y) for i in range(2)]
                    us = graph_per_launch(dev, fns)
                    rec(f"gemm_4bit_M{M}_{qt}_{dt}_{K}x{N}", us, nbw + 2 * M * K + 2 * M * N, 2 * M * N * K)
            del ps, as_

    # prefill forward and backward
    M0, K, N = PREFILL
    ps, as_ = qweight(N, K, 0.02, 0, "nf4", 2)
    for M in (512, 2048):
        X = synthetic.normal((M, K), 4000, 1.0, "bf16", device=d)
        dY = synthetic.normal((M, N), 5000, 1.0, "bf16", device=d)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        fl = 2 * M * N * K
        us = graph_per_launch(dev, [lambda i=i: b.gemm_4bit(X, ps[i], as_[i], N, None, BLOCK, "nf4", out=Y)
                                    for i in range(2)])
        rec(f"gemm_4bit_M{M}_nf4_bf16_{K}x{N}", us, wbytes(N, K) + 2 * M * K + 2 * M * N, fl)
        us = graph_per_launch(dev, [lambda i=i: b.gemm_4bit_backward(dY, ps[i], as_[i], K, BLOCK, "nf4", out=dX)
                                    for i in range(2)])
        rec(f"gemm_4bit_backward_M{M}_nf4_bf16_{K}x{N}", us, wbytes(N, K) + 2 * M * N + 2 * M * K, fl)
    del ps, as_
    out["note"] = ("each op alone: its launches back to back in one CUDA graph over rotating copies of its "
                   "inputs (the working set of a pass is above 5x L2, so every launch reads cold data); "
                   "time per launch = replay time / launches")
    return out


# ----------------------------------------------------------------- our arm

class Step:
    """Device buffers for one batch and the launch sequence of one step."""

    def __init__(self, dev, seed):
        import bit_blockwise_weight_b200 as bnb4
        import synthetic
        self.bnb4 = bnb4
        d = str(dev)
        self.x = synthetic.roundtrip_tensor(N_ELEMS, seed, "bf16", device=d)
        self.packed = torch.empty(N_ELEMS // 2, dtype=torch.uint8, device=dev)
        self.absmax = torch.empty(N_ELEMS // BLOCK, dtype=torch.float32, device=dev)
        self.deq = torch.empty(N_ELEMS, dtype=torch.bfloat16, device=dev)

        def qweight(N, K, sigma, s):
            w = synthetic.normal((N * K,), s, sigma, "f32", device=d)
            p, a = bnb4.quantize_4bit(w, BLOCK, "nf4")
            del w
            return p, a

        self.gemv = []
        for i, (K, N) in enumerate(GEMV_SHAPES):
            p, a = qweight(N, K, 0.02, 100 * seed + i)
            xv = synthetic.normal((K,), 1000 + seed, 1.0, "bf16", device=d)
            b = synthetic.normal((N,), 2000 + seed, 1.0, "bf16", device=d)
            self.gemv.append((K, N, p, a, xv, b, torch.empty(N, dtype=torch.bfloat16, device=dev)))
        self.smallm = []
        for i, (K, N) in enumerate(SMALLM_SHAPES):
            p, a = qweight(N, K, 0.015, 100 * seed + 10 + i)
            X = synthetic.normal((SMALLM_M, K), 3000 + seed + i, 1.0, "bf16", device=d)
            self.smallm.append((K, N, p, a, X,
                                torch.empty(SMALLM_M, N, dtype=torch.bfloat16, device=dev)))
        M, K, N = PREFILL
        p, a = qweight(N, K, 0.02, 100 * seed + 20)
        X = synthetic.normal((M, K), 4000 + seed, 1.0, "bf16", device=d)
        dY = synthetic.normal((M, N), 5000 + seed, 1.0, "bf16", device=d)
        self.prefill = (M, K, N, p, a, X, dY, torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                        torch.empty(M, K, dtype=torch.bfloat16, device=dev))
        torch.cuda.synchronize(dev)

    def launches(self):
        """The step as a list of zero-argument callables, one per kernel launch."""
        b = self.bnb4
        L = [lambda: b.quantize_4bit_into(self.x, self.packed, self.absmax, BLOCK, "nf4")]
        for K, N, p, a, xv, bias, y in self.gemv:
            L.append(lambda K=K, N=N, p=p, a=a, xv=xv, bias=bias, y=y:
                     b.gemv_4bit(xv, p, a, N, K, bias, BLOCK, "nf4", out=y))
        for K, N, p, a, X, Y in self.smallm:
            L.append(lambda N=N, p=p, a=a, X=X, Y=Y: b.gemm_4bit(X, p, a, N, None, BLOCK, "nf4", out=Y))
        M, K, N, p, a, X, dY, Y, dX = self.prefill
        L.append(lambda: b.gemm_4bit(X, p, a, N, None, BLOCK, "nf4", out=Y))
        L.append(lambda: b.gemm_4bit_backward(dY, p, a, K, BLOCK, "nf4", out=dX))
        L.append(lambda: b.dequantize_4bit(self.packed, self.absmax, N_ELEMS, BLOCK, "nf4", out=self.deq))
        return L


def run_ours(args, rank, world, dev):
    import bit_blockwise_weight_b200 as bnb4
    hbm, tc_burst, tc_sust, peak_kind = load_peaks()
    ops = step_ops()
    step = Step(dev, seed=rank)
    calls = step.launches()
    assert len(calls) == len(ops)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        for c in calls:
            c()
    torch.cuda.synchronize(dev)

    # The step's launches, captured once as a CUDA graph with a timing event
    # node after each launch, so that host launch latency does not leave the
    # GPU idle between the short kernels.  The launches (and the tensor maps
    # they carry) are exactly those of an eager step.
    # The timed graph holds the launches alone (an event node between two
    # kernels makes the second wait for the first to drain); a second graph
    # with the event nodes gives the per-launch breakdown.
    gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(calls) + 1)]
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    graph, graph_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        for c in calls:
            c()
    with torch.cuda.graph(graph_ev, stream=cap):
        gev[0].record(cap)
        for i, c in enumerate(calls):
            c()
            gev[i + 1].record(cap)
    torch.cuda.synchronize(dev)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
    t0.record(stream)
    for k in range(args.steps):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    if world > 1:
        torch.distributed.barrier()

    # per-launch durations: the same graph, the events read after each replay
    per_step = []
    for k in range(args.steps):
        graph_ev.replay()
        torch.cuda.synchronize(dev)
        per_step.append([gev[i].elapsed_time(gev[i + 1]) for i in range(len(calls))])
    # the clocks: sampled from just before the timed replays to the end of the
    # per-launch replays of the same graph that follow them
    clocks = sampler.stop() if sampler else None
    if clocks:
        clocks["window"] = "the timed replays and the per-launch replays after them"
    per_op_ms = [statistics.mean(st[i] for st in per_step) for i in range(len(calls))]
    del graph, graph_ev
    step_bytes = sum(b for _, b, _ in ops)
    value = job_rate(step_bytes, args.steps, world, ms) / 1e9

    # the next rows beyond the step (double-quantized statistics), timed on their own
    next_rows = time_next_rows(step, dev, hbm)
    next_rows.update(time_8bit_and_embedding(dev, hbm))
    configs = time_configs(dev, hbm, tc_burst, tc_sust)

    # e2e: the same step through the public API from pinned host buffers; the step's
    # inputs go host->device and every output comes back device->host, every step
    e2e = run_e2e(args, step, dev, stream, world)

    if rank != 0:
        return None
    roof, parts = roofline_and_parts(ops, per_op_ms, hbm, tc_burst, tc_sust, peak_kind)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) / N(0,0.02) tensors; no checkpoints)",
        "config": bench_config(world),
        "timing": "step captured once as a CUDA graph of its launches; K replays between two "
                  "events; per-launch times from a second graph with an event node after each "
                  "launch",
        "metric_values": metric_values(configs),
        "roofline": roof,
        "parts": parts,
        "configs_timed": configs,
        "next_rows": next_rows,
        "e2e": e2e,
        "gpu_launches": len(calls) * args.steps,
        "clocks": clocks,
        "library": bnb4.library_path(),
    }
    if args.cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    return line


def metric_values(configs):
    """The metric's own numbers, from the per-config timings: gemv_4bit on the
    gemv NF4 workload (4096 x 4096, no bias, bf16) in GB/s and as a fraction of
    the measured HBM copy bandwidth, and quantize_4bit of 2^28 elements (NF4,
    blocksize 64) in GB/s for the three input dtypes."""
    out = {}
    g = configs.get("gemv_4bit_nf4_bf16_4096x4096")
    if g:
        out["gemv_4bit_nf4_4096x4096"] = {k: g[k] for k in ("us", "GB/s", "hbm_frac")}
    for dt in ("bf16", "f16", "f32"):
        q = configs.get(f"quantize_4bit_2p28_{dt}_nf4_B64")
        if q:
            out[f"quantize_4bit_2p28_{dt}_nf4_B64"] = {k: q[k] for k in ("us", "GB/s", "hbm_frac")}
    return out


def time_next_rows(step, dev, hbm):
    """Double quantization of absmax and the gemv on 8-bit statistics, outside
    the step: double_quant / dequant_absmax of 2^22 absmax values (groups of
    256), and each gemv decode shape (with bias) on fp32 absmax and on its
    double-quantized absmax, side by side.  Each op timed with
    graph_per_launch over rotating copies of its inputs."""
    import bit_blockwise_weight_b200 as b
    G = 256
    n = step.absmax.numel()
    C = copies_for(5 * n)
    srcs = [step.absmax] + [step.absmax.clone() for _ in range(C - 1)]
    qs = [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(C)]
    ss = [torch.empty((n + G - 1) // G, dtype=torch.float32, device=dev) for _ in range(C)]
    backs = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(C)]
    for i in range(C):
        b.double_quant(srcs[i], G, out=(qs[i], ss[i]))
    out = {}

    def rec(name, us, nbytes):
        out[name] = {"us": round(us, 2), "bytes": int(nbytes), "GB/s": round(nbytes / (us / 1e6) / 1e9, 1),
                     "hbm_frac": round(nbytes / (us / 1e6) / 1e9 / hbm, 4)}

    rec("double_quant_absmax_4194304",
        graph_per_launch(dev, [lambda i=i: b.double_quant(srcs[i], G, out=(qs[i], ss[i])) for i in range(C)]),
        4 * n + n + 4 * ss[0].numel())
    rec("dequant_absmax_4194304",
        graph_per_launch(dev, [lambda i=i: b.dequant_absmax(qs[i], ss[i], G, out=backs[i]) for i in range(C)]),
        n + 4 * ss[0].numel() + 4 * n)
    del srcs, qs, ss, backs
    for K, N, p, a, xv, bias, y in step.gemv:
        nb = N * K // BLOCK
        C = copies_for(N * K // 2 + 4 * nb)
        ps = [p] + [p.clone() for _ in range(C - 1)]
        as_ = [a] + [a.clone() for _ in range(C - 1)]
        q8s, s8s = zip(*[b.double_quant(a_, G) for a_ in as_])
        rec(f"gemv_4bit_{K}x{N}", graph_per_launch(dev, [
            lambda i=i: b.gemv_4bit(xv, ps[i], as_[i], N, K, bias, BLOCK, "nf4", out=y) for i in range(C)]),
            N * K // 2 + 4 * nb + 2 * K + 4 * N)
        rec(f"gemv_4bit_dq_{K}x{N}", graph_per_launch(dev, [
            lambda i=i: b.gemv_4bit_dq(xv, ps[i], q8s[i], s8s[i], N, K, bias, BLOCK, "nf4", G, out=y)
            for i in range(C)]), N * K // 2 + nb + 4 * s8s[0].numel() + 2 * K + 4 * N)
        out[f"gemv_4bit_dq_{K}x{N}"]["speedup_vs_fp32_absmax"] = round(
            out[f"gemv_4bit_{K}x{N}"]["us"] / out[f"gemv_4bit_dq_{K}x{N}"]["us"], 3)
        del ps, as_, q8s, s8s
    # M >= 2 on 8-bit statistics: small-M M = 16 on the 70B shapes and prefill M = 512
    # forward / backward, each beside the same op on fp32 absmax
    for K, N, p, a, X, Y in step.smallm:
        q8, s8 = b.double_quant(a, G)
        nb = N * K // BLOCK
        ps = [p, p.clone()]
        as_ = [a, a.clone()]
        q8s, s8s = [q8, q8.clone()], [s8, s8.clone()]
        M = X.shape[0]
        rec(f"gemm_4bit_M{M}_{K}x{N}", graph_per_launch(dev, [
            lambda i=i: b.gemm_4bit(X, ps[i], as_[i], N, None, BLOCK, "nf4", out=Y) for i in range(2)]),
            N * K // 2 + 4 * nb + 2 * M * K + 2 * M * N)
        rec(f"gemm_4bit_dq_M{M}_{K}x{N}", graph_per_launch(dev, [
            lambda i=i: b.gemm_4bit_dq(X, ps[i], q8s[i], s8s[i], N, None, BLOCK, "nf4", G, out=Y) for i in range(2)]),
            N * K // 2 + nb + 4 * s8.numel() + 2 * M * K + 2 * M * N)
        out[f"gemm_4bit_dq_M{M}_{K}x{N}"]["speedup_vs_fp32_absmax"] = round(
            out[f"gemm_4bit_M{M}_{K}x{N}"]["us"] / out[f"gemm_4bit_dq_M{M}_{K}x{N}"]["us"], 3)
        del ps, as_, q8s, s8s
    M, K, N, p, a, X, dY, Y, dX = step.prefill
    q8, s8 = b.double_quant(a, G)
    for name, f32f, dqf in (
            (f"gemm_4bit_M{M}_{K}x{N}", lambda: b.gemm_4bit(X, p, a, N, None, BLOCK, "nf4", out=Y),
             lambda: b.gemm_4bit_dq(X, p, q8, s8, N, None, BLOCK, "nf4", G, out=Y)),
            (f"gemm_4bit_backward_M{M}_{K}x{N}", lambda: b.gemm_4bit_backward(dY, p, a, K, BLOCK, "nf4", out=dX),
             lambda: b.gemm_4bit_backward_dq(dY, p, q8, s8, K, BLOCK, "nf4", G, out=dX))):
        t32 = graph_per_launch(dev, [f32f] * 4)
        tdq = graph_per_launch(dev, [dqf] * 4)
        out[name] = {"us": round(t32, 2)}
        dqn = name.replace("gemm_4bit", "gemm_4bit_dq", 1)
        out[dqn] = {"us": round(tdq, 2), "speedup_vs_fp32_absmax": round(t32 / tdq, 3)}
    # fp32 compute dtype (x, bias and y in float32; CUDA-core FMAs on the exact
    # fp32 dequantized weight): the decode shapes, M = 16 on the 70B shapes and
    # prefill M = 512 forward / backward.  The prefill is compute-bound on the
    # CUDA cores: its fraction is of the fp32 FMA rate from the unit counts
    # (148 SMs x 128 lanes x 2 flops x the clock seen)
    fp32_peak = 148 * 128 * 2 * CLOCK_MHZ_NOMINAL * 1e6 / 1e12
    for K, N, p, a, xv, bias, y in step.gemv:
        nb = N * K // BLOCK
        C = copies_for(N * K // 2 + 4 * nb)
        ps = [p] + [p.clone() for _ in range(C - 1)]
        as_ = [a] + [a.clone() for _ in range(C - 1)]
        x32, b32 = xv.float(), bias.float()
        y32 = torch.empty(N, dtype=torch.float32, device=dev)
        rec(f"gemv_4bit_f32_{K}x{N}", graph_per_launch(dev, [
            lambda i=i: b.gemv_4bit(x32, ps[i], as_[i], N, K, b32, BLOCK, "nf4", out=y32) for i in range(C)]),
            N * K // 2 + 4 * nb + 4 * K + 8 * N)
        del ps, as_
    for K, N, p, a, X, Y in step.smallm:
        nb = N * K // BLOCK
        ps = [p, p.clone()]
        as_ = [a, a.clone()]
        M = X.shape[0]
        X32 = X.float()
        Y32 = torch.empty(M, N, dtype=torch.float32, device=dev)
        name = f"gemm_4bit_f32_M{M}_{K}x{N}"
        rec(name, graph_per_launch(dev, [
            lambda i=i: b.gemm_4bit(X32, ps[i], as_[i], N, None, BLOCK, "nf4", out=Y32) for i in range(2)]),
            N * K // 2 + 4 * nb + 4 * M * K + 4 * M * N)
        # at M = 16 the fp32 FMAs, not HBM, bound it: report both
        tf = 2.0 * M * N * K / (out[name]["us"] / 1e6) / 1e12
        out[name].update({"TFLOP/s": round(tf, 1), "fp32_fma_frac": round(tf / fp32_peak, 4)})
        del ps, as_
    M, K, N, p, a, X, dY, Y, dX = step.prefill
    X32, dY32 = X.float(), dY.float()
    Y32 = torch.empty(M, N, dtype=torch.float32, device=dev)
    dX32 = torch.empty(M, K, dtype=torch.float32, device=dev)
    flops = 2.0 * M * N * K
    for name, f in ((f"gemm_4bit_f32_M{M}_{K}x{N}", lambda: b.gemm_4bit(X32, p, a, N, None, BLOCK, "nf4", out=Y32)),
                    (f"gemm_4bit_backward_f32_M{M}_{K}x{N}",
                     lambda: b.gemm_4bit_backward(dY32, p, a, K, BLOCK, "nf4", out=dX32))):
        us = graph_per_launch(dev, [f] * 2, reps=2)
        tf = flops / (us / 1e6) / 1e12
        out[name] = {"us": round(us, 2), "TFLOP/s": round(tf, 1), "fp32_fma_frac": round(tf / fp32_peak, 4)}
    out["note"] = ("each op alone, back to back in one CUDA graph over rotating copies of its inputs "
                   "(working set above 5x L2; the prefill ops reuse one 33 MB weight, compute-bound)")
    return out


def code8_table(seed: int = 0):
    """A seeded 256-entry table for the 8-bit rows: -1, 0, 1 and magnitudes spread
    log-uniformly down to 2^-24 (a wide dynamic range), strictly ascending."""
    import numpy as np
    rng = np.random.default_rng(seed)
    vals = {-1.0, 0.0, 1.0}
    while len(vals) < 256:
        v = float(np.float32(rng.choice([-1.0, 1.0]) * 2.0 ** rng.uniform(-24.0, 0.0)))
        if v == 0.0 or abs(v) >= 2.0 ** -24:
            vals.add(v)
    return torch.tensor(sorted(vals), dtype=torch.float32)


def time_8bit_and_embedding(dev, hbm):
    """Rows f3 and f4 outside the step: quantize_8bit / dequantize_8bit of 2^26
    bf16 elements (B 64, a seeded log-spread table), and 4096 embedding lookups
    in a 128256 x 4096 NF4 table (B 64) to bf16.  Each op timed with
    graph_per_launch (the 8-bit inputs rotate over 3 copies, 600 MB; the
    lookups read 43 MB of a 263 MB table at random rows)."""
    import bit_blockwise_weight_b200 as b
    import synthetic
    d = str(dev)
    n = 1 << 26
    code = code8_table(0)
    C = 3
    xs = [synthetic.roundtrip_tensor(n, i, "bf16", device=d) for i in range(C)]
    qs = [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(C)]
    a8s = [torch.empty(n // BLOCK, dtype=torch.float32, device=dev) for _ in range(C)]
    y8 = torch.empty(n, dtype=torch.bfloat16, device=dev)
    stream = lambda: torch.cuda.current_stream(dev).cuda_stream
    out = {}

    def rec(name, us, nbytes):
        out[name] = {"us": round(us, 2), "bytes": int(nbytes), "GB/s": round(nbytes / (us / 1e6) / 1e9, 1),
                     "hbm_frac": round(nbytes / (us / 1e6) / 1e9 / hbm, 4)}

    rec("quantize_8bit_2p26_bf16", graph_per_launch(dev, [
        lambda i=i: b.bnb4_quantize_8bit(xs[i].data_ptr(), qs[i].data_ptr(), a8s[i].data_ptr(), n, BLOCK,
                                         code.data_ptr(), 2, stream()) for i in range(C)]),
        2 * n + n + 4 * (n // BLOCK))
    rec("dequantize_8bit_2p26_bf16", graph_per_launch(dev, [
        lambda i=i: b.bnb4_dequantize_8bit(qs[i].data_ptr(), a8s[i].data_ptr(), y8.data_ptr(), n, BLOCK,
                                           code.data_ptr(), 2, stream()) for i in range(C)]),
        n + 4 * (n // BLOCK) + 2 * n)
    del xs, qs, a8s, y8
    V, D, T = 128256, 4096, 4096
    w = synthetic.normal((V * D,), 7, 0.02, "f32", device=d)
    ep, ea = b.quantize_4bit(w, BLOCK, "nf4")
    del w
    g = torch.Generator(device=d).manual_seed(11)
    idxs = [torch.randint(0, V, (T,), generator=g, device=d, dtype=torch.int64) for _ in range(8)]
    eo = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    rec("embedding_4bit_4096_of_128256x4096", graph_per_launch(dev, [
        lambda i=i: b.embedding_4bit(ep, ea, V, D, idxs[i], BLOCK, "nf4", out=eo) for i in range(8)]),
        T * (D // 2 + 4 * (D // BLOCK)) + 8 * T + 2 * T * D)
    return out


def run_e2e(args, step, dev, stream, world=1):
    """Same step, host buffers in and out through the public API (pinned memory);
    whole-job rate over the slowest rank (every rank calls this).

    Every step copies its inputs host->device, runs the step's launches and
    copies every output device->host.  Consecutive steps are pipelined the way
    a serving loop would run them: two sets of device buffers, the host->device
    copies on one copy stream and the device->host copies on another, so step
    i+1's inputs and step i-1's outputs cross PCIe (full duplex) while step i
    computes.  Each set's inputs are not overwritten before its previous step
    has read them, nor its outputs before they have been copied out.  The timed
    region runs from before the first input copy to after the last output copy.
    """
    import bit_blockwise_weight_b200 as bnb4
    h_x = step.x.cpu().pin_memory()
    h_gemv_x = [g[4].cpu().pin_memory() for g in step.gemv]
    h_sm_X = [s[4].cpu().pin_memory() for s in step.smallm]
    M, K, N, p, a, X, dY, Y, dX = step.prefill
    h_X, h_dY = X.cpu().pin_memory(), dY.cpu().pin_memory()

    def buffers(st):
        outs = [st.packed, st.absmax, st.deq] + [g[6] for g in st.gemv] + [s[5] for s in st.smallm] + \
            [st.prefill[7], st.prefill[8]]
        ins = [(h_x, st.x)] + [(h, g[4]) for h, g in zip(h_gemv_x, st.gemv)] + \
            [(h, s[4]) for h, s in zip(h_sm_X, st.smallm)] + [(h_X, st.prefill[5]), (h_dY, st.prefill[6])]
        return ins, outs, st.launches()

    sets = [buffers(step), buffers(Step(dev, seed=int(os.environ.get("RANK", "0"))))]
    h_outs = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in sets[0][1]]
    h2d = sum(h.numel() * h.element_size() for h, _ in sets[0][0])
    d2h = sum(o.numel() * o.element_size() for o in sets[0][1])
    steps = max(2, min(args.steps, 8))
    c_in, c_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def one(i):
        k = i % 2
        ins, outs, calls = sets[k]
        with torch.cuda.stream(c_in):
            if started[k]:
                c_in.wait_event(ev_comp[k])    # the set's previous step has read its inputs
            for h, d in ins:
                d.copy_(h, non_blocking=True)
            ev_in[k].record(c_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[k])
            if started[k]:
                stream.wait_event(ev_out[k])   # the set's previous outputs are out
            for c in calls:
                c()
            ev_comp[k].record(stream)
        with torch.cuda.stream(c_out):
            c_out.wait_event(ev_comp[k])
            for h, o in zip(h_outs, outs):
                h.copy_(o, non_blocking=True)
            ev_out[k].record(c_out)
        started[k] = True

    def run(n, begin=None):
        if begin is not None:
            c_in.wait_event(begin)
        for i in range(n):
            one(i)
        for k in range(2):
            if started[k]:
                stream.wait_event(ev_out[k])

    run(2)   # warm-up: both sets once
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(steps, begin=e0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    step_bytes = sum(b for _, b, _ in step_ops())
    return {"value": round(job_rate(step_bytes, steps, world, ms) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world, "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "pipelining": "two buffer sets; inputs in on one copy stream and outputs out on another "
                          "overlap the neighbouring steps' compute"}


# ------------------------------------------------------------ CPU oracle arm

def oracle_sample(seed: int = 0):
    """Time the CPU oracle on a bounded sample of every op of the step.

    Returns (extrapolated GB/s for the whole step, extrapolated seconds per
    step, per-op detail).  Each op runs on a slice of its workload (a number
    of elements, rows or output entries); its time is scaled to the full op
    by that fraction.  `seed` picks the slice's inputs.
    """
    import numpy as np
    import oracle
    import synthetic
    oracle.lib()
    ops = step_ops()
    detail = {}
    full_time = 0.0
    frac_q = 1 << 24
    x = synthetic.storage_numpy(synthetic.roundtrip_tensor(frac_q, seed, "bf16"))
    t = time.perf_counter()
    p, a = oracle.quantize(x, "bf16", BLOCK, "nf4")
    tq = (time.perf_counter() - t) * (N_ELEMS / frac_q)
    t = time.perf_counter()
    oracle.dequantize(p, a, frac_q, BLOCK, "nf4", "bf16")
    td = (time.perf_counter() - t) * (N_ELEMS / frac_q)
    detail["quantize_4bit"] = f"{frac_q} elements"
    detail["dequantize_4bit"] = f"{frac_q} elements"
    full_time += tq + td

    def mm_rows(K, N, M, rows, backward=False):
        w = synthetic.weight(min(N, 64), K, seed).numpy().reshape(-1)
        wp, wa = oracle.quantize(w, "f32", BLOCK, "nf4")
        Nw = min(N, 64)
        if backward:
            dY = synthetic.storage_numpy(synthetic.grad_output(1, Nw, 3)).reshape(-1)
            ks = np.arange(rows) % K
            t = time.perf_counter()
            oracle.matmul_backward_entries(dY, "bf16", wp, wa, 1, Nw, K, BLOCK, "nf4",
                                           np.zeros(rows, np.int64), ks)
            el = time.perf_counter() - t
            return el / rows * (N / Nw) * (M * K)   # each entry sums over N
        X = synthetic.storage_numpy(synthetic.activations(1, K, 1)).reshape(-1)
        js = np.arange(rows) % Nw
        t = time.perf_counter()
        oracle.matmul_entries(X, "bf16", wp, wa, None, 1, Nw, K, BLOCK, "nf4",
                              np.zeros(rows, np.int64), js)
        el = time.perf_counter() - t
        return el / rows * (M * N)

    for K, N in GEMV_SHAPES:
        full_time += mm_rows(K, N, 1, 2048)
        detail[f"gemv_4bit_{K}x{N}"] = "2048 output entries"
    for K, N in SMALLM_SHAPES:
        full_time += mm_rows(K, N, SMALLM_M, 2048)
        detail[f"gemm_4bit_M{SMALLM_M}_{K}x{N}"] = "2048 output entries"
    M, K, N = PREFILL
    full_time += mm_rows(K, N, M, 2048)
    full_time += mm_rows(K, N, M, 16384, backward=True)
    detail["prefill"] = "2048 forward and 16384 backward output entries (64-row weight slice)"
    step_bytes = sum(b for _, b, _ in ops)
    return step_bytes / full_time / 1e9, full_time, detail


def oracle_all_cores(threads=None):
    """The oracle on every host core at once: one thread per core, each timing
    its own slice of every op (the C oracle runs through ctypes, which releases
    the GIL for the call).  Returns (whole-step GB/s over all threads, threads,
    mean extrapolated seconds per step and thread)."""
    import concurrent.futures as cf
    threads = threads or os.cpu_count() or 1
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        res = list(ex.map(oracle_sample, range(threads)))
    per_thread_s = statistics.mean(r[1] for r in res)
    step_bytes = sum(b for _, b, _ in step_ops())
    return threads * step_bytes / per_thread_s / 1e9, threads, per_thread_s


def cpu_baseline(measured=None):
    gbs, threads, per_thread_s = measured or oracle_all_cores()
    return {"value": round(gbs, 6), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": (f"the C oracle on {threads} host threads at once (one per core), each on its "
                       "own slice of every op of the step (2^24 quantize/dequantize elements, "
                       "2048-16384 output entries per matmul), each slice's time scaled to the "
                       f"full step ({round(per_thread_s, 1)} s per step and thread, extrapolated); "
                       "value = all threads' steps over that time"),
            "host_nproc": os.cpu_count()}


def bench_config(world):
    return {"workload": WORKLOAD, "n_elems": N_ELEMS, "quant_type": "nf4",
            "blocksize": BLOCK, "gemv_shapes_KN": GEMV_SHAPES,
            "smallm": {"M": SMALLM_M, "shapes_KN": SMALLM_SHAPES},
            "prefill_MKN": PREFILL, "parallelism": f"dp{world} (independent batches)",
            "l2": "inputs larger than L2 (step working set ~1.6 GB vs 126 MB L2)"}


def run_reference(args):
    """The reference arm: the CPU oracle on every host core, timed on bounded
    samples of the workload (one sample per step)."""
    for _ in range(args.warmup):
        oracle_all_cores()
    t = time.perf_counter()
    runs = [oracle_all_cores() for _ in range(args.steps)]
    wall = time.perf_counter() - t
    v = statistics.mean(r[0] for r in runs)
    base = cpu_baseline((v, runs[0][1], statistics.mean(r[2] for r in runs)))
    return {"metric": METRIC, "value": round(v, 6), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(wall / args.steps * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": bench_config(1),
            "cpu_baseline": base,
            "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


PROFILE_CASES = {
    # name: what runs (inputs above L2 size, a few hundred MB on the device at most)
    "quantize": "quantize_4bit, 2^26 bf16 elements, NF4, B=64",
    "quantize_fp4": "quantize_4bit, 2^26 bf16 elements, FP4, B=64",
    "dequantize": "dequantize_4bit, 2^26 elements to bf16, NF4, B=64",
    "gemv": "gemv_4bit + bias, K=4096, N=14336, NF4 B=64, bf16",
    "gemm_small": "gemm_4bit M=16, K=8192, N=28672, NF4 B=64, bf16",
    "gemm_tc": "gemm_4bit M=512, K=4096, N=14336, NF4 B=64, bf16",
    "gemm_tc_backward": "gemm_4bit_backward M=512, K=4096, N=14336, NF4 B=64, bf16",
    "double_quant": "double_quant + dequant_absmax of 2^25 absmax values, groups of 256",
    "gemv_dq": "gemv_4bit_dq + bias, K=4096, N=14336, NF4 B=64, double-quantized absmax "
               "(groups of 256), bf16",
    "gemm_f32_small": "gemm_4bit M=16, K=8192, N=28672, NF4 B=64, fp32",
}


def profile_case(name):
    """One launch of one kernel on a small case, for an ncu capture (no timing, no JSON line).

    Setup launches (input draws, weight quantization) come first; the kernel of
    interest is the last launch of its kind."""
    import bit_blockwise_weight_b200 as bnb4
    import synthetic
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = str(dev)
    if name in ("quantize", "dequantize", "quantize_fp4"):
        x = synthetic.roundtrip_tensor(1 << 26, 0, "bf16", device=d)
        p, a = bnb4.quantize_4bit(x, BLOCK, "fp4" if name == "quantize_fp4" else "nf4")
        if name == "dequantize":
            bnb4.dequantize_4bit(p, a, x.numel(), BLOCK, "nf4", dtype=torch.bfloat16)
    elif name == "double_quant":
        a = synthetic.absmax_values(1 << 25, seed=4).to(dev)
        q, s = bnb4.double_quant(a, 256)
        bnb4.dequant_absmax(q, s, 256)
    else:
        K, N, M = {"gemv": (4096, 14336, 1), "gemv_dq": (4096, 14336, 1), "gemm_small": (8192, 28672, 16),
                   "gemm_f32_small": (8192, 28672, 16), "gemm_tc": (4096, 14336, 512),
                   "gemm_tc_backward": (4096, 14336, 512)}[name]
        w = synthetic.normal((N * K,), 0, 0.02, "f32", device=d)
        p, a = bnb4.quantize_4bit(w, BLOCK, "nf4")
        del w
        if name == "gemv":
            bnb4.gemv_4bit(synthetic.normal((K,), 1, 1.0, "bf16", device=d), p, a, N, K,
                           synthetic.normal((N,), 2, 1.0, "bf16", device=d))
        elif name == "gemv_dq":
            q8, s8 = bnb4.double_quant(a, 256)
            bnb4.gemv_4bit_dq(synthetic.normal((K,), 1, 1.0, "bf16", device=d), p, q8, s8, N, K,
                              synthetic.normal((N,), 2, 1.0, "bf16", device=d))
        elif name == "gemm_f32_small":
            bnb4.gemm_4bit(synthetic.normal((M, K), 1, 1.0, "f32", device=d), p, a, N)
        elif name == "gemm_tc_backward":
            bnb4.gemm_4bit_backward(synthetic.normal((M, N), 3, 1.0, "bf16", device=d), p, a, K)
        else:
            bnb4.gemm_4bit(synthetic.normal((M, K), 1, 1.0, "bf16", device=d), p, a, N)
    torch.cuda.synchronize(dev)
    print(f"profile case {name}: {PROFILE_CASES[name]}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="run one launch of one kernel on a small case for an ncu capture "
                         "(prints no bench line)")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    args.cpu_baseline = args.cpu_baseline and rank == 0 and world == 1
    line = run_ours(args, rank, world, dev)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
