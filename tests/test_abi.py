"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host (no GPU needed: every check below returns
before anything is enqueued)."""
import ctypes
import os
import re

import pytest

import bit_blockwise_weight_b200 as bnb4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"\b(bnb4_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_calls():
    names = declared_functions()
    for want in ("bnb4_quantize", "bnb4_dequantize", "bnb4_gemv", "bnb4_gemm",
                 "bnb4_gemm_backward", "bnb4_status_string", "bnb4_version"):
        assert want in names


@pytest.mark.parametrize("name", declared_functions())
def test_library_exports_every_declared_symbol(name):
    lib = ctypes.CDLL(bnb4.library_path())
    assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings_and_version():
    assert bnb4.bnb4_version() >= 10000
    for s in range(11):
        assert bnb4.status_string(s) != "unknown status"
    assert bnb4.status_string(0) == "ok"
    assert bnb4.status_string(99) == "unknown status"


A = 4096  # a fake 16-byte aligned address; never dereferenced: validation fails first


def test_quantize_argument_checks():
    q = bnb4.bnb4_quantize
    assert q(A, A, A, -1, 64, 0, 0, None) == 4          # negative n
    assert q(A, A, A, 10, 32, 0, 0, None) == 3          # blocksize too small
    assert q(A, A, A, 10, 96, 0, 0, None) == 3          # not a power of two
    assert q(A, A, A, 10, 8192, 0, 0, None) == 3        # too large
    assert q(A, A, A, 10, 64, 2, 0, None) == 6          # quant type
    assert q(A, A, A, 10, 64, 0, 3, None) == 5          # dtype
    assert q(None, A, A, 10, 64, 0, 0, None) == 1       # null
    assert q(A + 2, A, A, 10, 64, 0, 0, None) == 2      # misaligned
    assert q(None, None, None, 0, 64, 0, 0, None) == 0  # n == 0: nothing to do


def test_dequantize_argument_checks():
    d = bnb4.bnb4_dequantize
    assert d(A, A, None, 10, 64, 0, 2, None) == 1
    assert d(A, A + 8, A, 10, 64, 0, 2, None) == 2
    assert d(A, A, A, 10, 64, 1, 7, None) == 5
    assert d(A, A, A, 10, 100, 1, 2, None) == 3


def test_matmul_argument_checks():
    g = bnb4.bnb4_gemv
    assert g(A, A, A, None, A, 128, 100, 64, 0, 2, None) == 4   # K % 32
    assert g(A, A, A, None, A, 128, 96, 64, 0, 2, None) == 4    # K % blocksize
    assert g(A, A, A, None, A, 0, 128, 64, 0, 2, None) == 4     # N < 1
    assert g(A, A, A, None, A, 128, 128, 64, 0, 7, None) == 5   # not a dtype
    assert bnb4.bnb4_gemv_dq(A, A, A, A, 256, None, A, 128, 128, 64, 0, 0, None) == 5  # no f32 on 8-bit statistics
    assert g(A, A, A, A + 4, A, 128, 128, 64, 0, 2, None) == 2  # misaligned bias
    assert g(A, None, A, None, A, 128, 128, 64, 0, 2, None) == 1
    m = bnb4.bnb4_gemm
    assert m(A, A, A, None, A, 0, 128, 128, 64, 0, 2, None) == 4
    assert m(A, A, A, None, A, 4, 128, 128, 64, 5, 2, None) == 6
    b = bnb4.bnb4_gemm_backward
    assert b(A, A, A, A, 4, 128, 100, 64, 0, 2, None) == 4
    assert b(A, A, A, None, 4, 128, 128, 64, 0, 2, None) == 1


def _code(values):
    import numpy as np
    c = np.ascontiguousarray(values, np.float32)
    return c, c.ctypes.data


def test_8bit_argument_checks():
    import numpy as np
    good, gp = _code((np.arange(256) - 128) / 128.0)
    for bad_vals in (np.arange(256)[::-1] / 255.0,                          # descending
                     np.where(np.arange(256) == 0, 2.0, np.linspace(-1, 1, 256)),   # out of range
                     np.where(np.arange(256) == 128, 1e-30, (np.arange(256) - 128) / 128.0),  # tiny entry
                     np.where(np.arange(256) == 5, np.nan, np.linspace(-1, 1, 256))):
        bad, bp = _code(bad_vals)
        assert bnb4.bnb4_quantize_8bit(A, A, A, 10, 64, bp, 0, None) == 9
        assert bnb4.bnb4_dequantize_8bit(A, A, A, 10, 64, bp, 2, None) == 9
    q = bnb4.bnb4_quantize_8bit
    assert q(A, A, A, 10, 64, None, 0, None) == 1        # no table
    assert q(A, A, A, 10, 32, gp, 0, None) == 3
    assert q(A, A, A, 10, 64, gp, 4, None) == 5
    assert q(A, A, A, -3, 64, gp, 0, None) == 4
    assert q(A, A + 1, A, 10, 64, gp, 0, None) == 2
    assert q(None, None, None, 0, 64, gp, 0, None) == 0  # n == 0: nothing to do
    d = bnb4.bnb4_dequantize_8bit
    assert d(A, None, A, 10, 64, gp, 2, None) == 1
    assert d(A, A, A + 8, 10, 64, gp, 2, None) == 2
    assert good.size == 256


def test_embedding_argument_checks():
    e = bnb4.bnb4_embedding_4bit
    assert e(A, A, 100, 64, 64, 0, A, 0, A, 2, None) == 0     # no indices: nothing to do
    assert e(A, A, 100, 0, 64, 0, A, 5, A, 2, None) == 4      # D < 1
    assert e(A, A, -1, 64, 64, 0, A, 5, A, 2, None) == 4      # V < 0
    assert e(A, A, 100, 64, 48, 0, A, 5, A, 2, None) == 3
    assert e(A, A, 100, 64, 64, 3, A, 5, A, 2, None) == 6
    assert e(A, A, 100, 64, 64, 0, A, 5, A, 7, None) == 5
    assert e(A, A, 100, 64, 64, 0, None, 5, A, 2, None) == 1
    assert e(A, A, 100, 64, 64, 0, A + 8, 5, A, 2, None) == 2


def test_header_is_plain_c_and_links(tmp_path):
    """include/bnb4.h compiles as C99 with warnings as errors; a C client links
    libbnb4.so and gets the documented host-side results."""
    import shutil
    import subprocess
    cc = shutil.which("cc") or shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = bnb4.library_path()
    exe = tmp_path / "c_abi_check"
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe),
                           lib, "-Wl,-rpath," + os.path.dirname(lib)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert "c abi ok" in out.stdout


def test_product_package_does_not_use_the_oracle():
    """The product never imports, includes, links or loads anything under oracle/."""
    pkg = os.path.join(ROOT, "bit_blockwise_weight_b200")
    bad = re.compile(r"(import\s+oracle|from\s+oracle|#include\s*[<\"][^>\"]*oracle|"
                     r"bnb4_oracle|liboracle)")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not bad.search(src), f
