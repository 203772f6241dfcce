"""The benchmark's JSON contract on the CPU: the reference arm's line (the
CPU oracle on bounded samples) and the roofline / per-op summary of our arm,
computed from given durations."""
import types

import pytest

import bench


def test_step_ops_cover_every_launch_once():
    ops = bench.step_ops()
    names = [n for n, _, _ in ops]
    assert len(names) == len(set(names)) == 10
    assert names[0] == "quantize_4bit" and names[-1] == "dequantize_4bit"
    n, B = bench.N_ELEMS, bench.BLOCK
    assert ops[0][1] == 2 * n + n // 2 + 4 * (n // B)        # bf16 in, packed and absmax out
    assert ops[-1][1] == n // 2 + 4 * (n // B) + 2 * n       # packed and absmax in, bf16 out
    for name, nbytes, flops in ops[1:-1]:
        assert nbytes > 0 and flops > 0


def test_roofline_and_parts():
    ops = [("quantize_4bit", 6_000_000, 0), ("gemm_4bit_M512_4096x14336", 40_000_000, 60_129_542_144),
           ("gemv_4bit_4096x4096", 9_000_000, 33_554_432)]
    roof, parts = bench.roofline_and_parts(ops, [0.002, 0.080, 0.010], 6500.0, 1683.5, 1400.0, "measured",
                                           traffic=lambda name: 123)
    # the tensor-core op has the largest share: TFLOP/s against the burst peak,
    # the sustained fraction beside it
    assert roof["bound"] == "tensor" and roof["kernel"] == "gemm_4bit_M512_4096x14336"
    assert roof["achieved"] == pytest.approx(60_129_542_144 / 80e-6 / 1e12, abs=0.1)
    assert roof["peak"] == 1683.5
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1683.5, abs=1e-4)
    assert roof["frac_of_sustained"] == pytest.approx(roof["achieved"] / 1400.0, abs=1e-4)
    assert roof["traffic"] == 123 and roof["unit"] == "TFLOP/s"
    assert sum(p["share"] for p in parts.values()) == pytest.approx(1.0, abs=1e-3)
    assert parts["quantize_4bit"]["GB/s"] == pytest.approx(6e6 / 2e-6 / 1e9, abs=0.1)
    roof, _ = bench.roofline_and_parts(ops[:1] + ops[2:], [0.5, 0.01], 6500.0, 1683.5, 1400.0, "measured",
                                       traffic=lambda name: None)
    assert roof["bound"] == "hbm" and roof["peak"] == 6500.0 and roof["traffic"] is None
    assert roof["frac"] == pytest.approx(6e6 / 0.5e-3 / 1e9 / 6500.0, abs=1e-4)


def test_reference_line():
    line = bench.run_reference(types.SimpleNamespace(steps=1, warmup=0))
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == bench.WORKLOAD


def test_reference_line_has_our_config():
    """Both arms describe the same workload with the same config dict."""
    assert bench.bench_config(1) == bench.bench_config(1)
    line = bench.run_reference(types.SimpleNamespace(steps=1, warmup=0))
    assert line["config"] == bench.bench_config(1)


def test_reference_arm_loads_no_product_library():
    """The reference arm (the oracle on the host cores) imports neither the
    product package nor its shared library."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, types; sys.path.insert(0, %r); import bench; "
            "bench.oracle_sample(0); "
            "assert 'bit_blockwise_weight_b200' not in sys.modules, 'product package imported'; "
            "maps = open('/proc/self/maps').read(); "
            "assert 'libbnb4' not in maps, 'libbnb4.so mapped'; print('ok')" % root)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr
