"""Write roundtrip_2p28_digests.json: SHA-256 digests of the CPU oracle's
outputs for every run of the full-size round-trip sweep.

The sweep: 1-D tensors of 2^28 elements drawn by synthetic.roundtrip_tensor
(N(0, 1) with 1% of the entries scaled by 20), seeds 0..3, in fp32 / fp16 /
bf16; NF4 and FP4; blocksizes 64 ... 4096.  For each of the 168 runs the
oracle quantizes the tensor (packed bytes, fp32 absmax) and dequantizes it
back to the input dtype; the digests are of the raw little-endian bytes of
those three arrays.  A GPU test recomputes the same arrays with the CUDA path
and compares digests, so every output element of every run is checked, not a
sample.

This calls only oracle/ and the seeded input generator; nothing from the CUDA
path.  Usage: python tests/golden/make_roundtrip_digests.py [--jobs N]
(about 18 s of oracle time per run; the runs are spread over N processes).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import multiprocessing as mp
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
OUT = os.path.join(HERE, "roundtrip_2p28_digests.json")

N_ELEMS = 1 << 28
SEEDS = (0, 1, 2, 3)
DTYPES = ("f32", "f16", "bf16")
QTYPES = ("nf4", "fp4")
BLOCKS = (64, 128, 256, 512, 1024, 2048, 4096)


def run_key(dt, qt, B, seed):
    return f"{dt}/{qt}/B{B}/seed{seed}"


def digest(a) -> str:
    return hashlib.sha256(memoryview(a).cast("B")).hexdigest()


def one_input(job):
    """All (quant type, blocksize) runs of one (seed, dtype) input."""
    seed, dt = job
    sys.path.insert(0, ROOT)
    import oracle
    import synthetic
    x = synthetic.storage_numpy(synthetic.roundtrip_tensor(N_ELEMS, seed, dt))
    out = {}
    for qt in QTYPES:
        for B in BLOCKS:
            packed, absmax = oracle.quantize(x, dt, B, qt)
            deq = oracle.dequantize(packed, absmax, N_ELEMS, B, qt, dt)
            out[run_key(dt, qt, B, seed)] = {"packed": digest(packed), "absmax": digest(absmax),
                                              "dequant": digest(deq)}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=os.cpu_count() or 1)
    args = ap.parse_args()
    jobs = [(s, dt) for s in SEEDS for dt in DTYPES]
    runs = {}
    with mp.get_context("spawn").Pool(min(args.jobs, len(jobs))) as pool:
        for res in pool.imap_unordered(one_input, jobs):
            runs.update(res)
    doc = {"n": N_ELEMS, "seeds": list(SEEDS), "dtypes": list(DTYPES), "quant_types": list(QTYPES),
           "blocksizes": list(BLOCKS),
           "inputs": "synthetic.roundtrip_tensor(2^28, seed, dtype): N(0,1), 1% x20 outliers",
           "arrays": "sha256 of packed (uint8), absmax (float32) and dequantize to the input dtype "
                     "(raw little-endian bytes)",
           "runs": dict(sorted(runs.items()))}
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    print(f"{len(runs)} runs -> {OUT}")


if __name__ == "__main__":
    main()
