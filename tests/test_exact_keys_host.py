"""The quantize kernel's exact-screen keys, as the library's host code builds them.

For FP4 with bf16 and fp16 inputs and NF4 with bf16 inputs the kernel decides
each element by the sign of x * RN(1/a) - key alone.  That is exact when every
ratio x / a of two such values (|x| <= a) that falls in a threshold's cell
lies further than |x / a| 2^-24 from the key, on the side where the IEEE
quotient RN(x / a) puts it: above the key exactly when the nearest code of
RN(x / a) (ties to the smaller index) is the upper one.  Checked here for every
ratio of significands near every threshold, against the keys printed by a
host-only build of the library's table code (tests/exact_keys_dump.cu); NF4
with fp16 inputs must be refused (its ratios come too close).
"""
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_blockwise_weight_b200", "csrc")


def f32(bits_hex):
    return float(np.array([int(bits_hex, 16)], np.uint32).view(np.float32)[0])


@pytest.fixture(scope="module")
def tables(tmp_path_factory):
    sys.path.insert(0, os.path.join(ROOT, "bit_blockwise_weight_b200"))
    import build  # noqa: E402
    nvcc = build.nvcc() if hasattr(build, "nvcc") else shutil.which("nvcc")
    if not nvcc or not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    exe = tmp_path_factory.mktemp("keys") / "exact_keys_dump"
    subprocess.check_call([nvcc, "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "exact_keys_dump.cu"), os.path.join(CSRC, "tables.cu"),
                           "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120, check=True).stdout
    cases, cur = {}, None
    for line in out.splitlines():
        f = line.split()
        if f[0] == "case":
            cur = cases[f[1]] = {"ok": f[2] == "1", "cells": []}
        elif f[0] == "codes":
            cur["codes"] = [f32(h) for h in f[1:]]
        elif f[0] == "cell":
            cur["cells"].append((int(f[1]), f32(f[2]), f32(f[3]), int(f[4])))
    return cases


def ratios(p):
    """Every X / A with X < 2^p and A in [2^(p-1), 2^p): the significand ratios."""
    A = np.arange(1 << (p - 1), 1 << p, dtype=np.float64)
    X = np.arange(0, 1 << p, dtype=np.float64)
    return np.unique((X[None, :] / A[:, None]).ravel())


def check_case(case, p):
    assert case["ok"]
    codes = np.array(case["codes"], np.float64)
    R = ratios(p)
    for k, key, thr, lohi in case["cells"]:
        lo, hi = lohi & 15, lohi >> 4
        c_lo, c_hi = codes[lo], codes[hi]
        mid = (c_lo + c_hi) / 2
        for d in range(0, -12, -1):           # x / a = (X / A) 2^d
            rho = R * 2.0 ** d
            rho = rho[np.abs(rho - abs(mid)) < 0.02 * abs(mid) + 1e-12]
            if rho.size == 0:
                continue
            rho = np.sign(mid) * rho          # the threshold's sign: x negative
            v = rho.astype(np.float32).astype(np.float64)   # RN32(x / a): exact for p <= 11
            dl, dh = np.abs(v - c_lo), np.abs(v - c_hi)
            upper = (dh < dl) | ((dh == dl) & (hi < lo))     # nearest code, ties to the smaller index
            assert np.array_equal(upper, rho > key), (k, d)
            assert np.all(np.abs(rho - key) > np.abs(rho) * 2.0 ** -24), (k, d)


def test_fp4_bf16_keys(tables):
    check_case(tables["fp4_bf16"], 8)


def test_fp4_f16_keys(tables):
    check_case(tables["fp4_f16"], 11)


def test_nf4_bf16_keys(tables):
    check_case(tables["nf4_bf16"], 8)


def test_nf4_f16_is_refused(tables):
    assert not tables["nf4_f16"]["ok"]
