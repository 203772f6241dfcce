"""CPU oracle for 4-bit blockwise weight quantization and the 4-bit matmuls.

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the
benchmark's CPU-baseline leg import this package.  Nothing in the product
package (``bit_blockwise_weight_b200``) imports it.  It shares no code,
header, table or constant with the CUDA library.

The arithmetic lives in plain C (``bnb4_oracle.c``, built to
``liboracle.so`` by :func:`build`).  This module only marshals numpy arrays.
``bruteforce.py`` holds an exact rational restatement for tiny inputs that
pins the C code.

16-bit data (fp16 / bf16) is passed as ``np.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bnb4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

QTYPES = {"nf4": 0, "fp4": 1}
DTYPES = {"f32": 0, "f16": 1, "bf16": 2}
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with the host C compiler (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "bnb4_oracle.h"))
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["cc", "-O1", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
             "-fexcess-precision=standard", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        sig = {
            "oracle_code_table": (I, [I, P]),
            "oracle_to_f32_array": (I, [P, I, I64, P]),
            "oracle_from_f32_array": (I, [P, I64, I, P]),
            "oracle_quantize": (I, [P, I, I64, I, I, P, P]),
            "oracle_dequantize": (I, [P, P, I64, I, I, I, P]),
            "oracle_matmul": (I, [P, I, P, P, P, I64, I64, I64, I, I, P]),
            "oracle_matmul_entries": (I, [P, I, P, P, P, I64, I64, I64, I, I, P, P, I64, P]),
            "oracle_matmul_backward": (I, [P, I, P, P, I64, I64, I64, I, I, P]),
            "oracle_matmul_backward_entries": (I, [P, I, P, P, I64, I64, I64, I, I, P, P, I64, P]),
            "oracle_double_quant": (I, [P, I64, I, P, P]),
            "oracle_dequant_absmax": (I, [P, P, I64, I, P]),
            "oracle_quantize_8bit": (I, [P, I, I64, I, P, P, P]),
            "oracle_dequantize_8bit": (I, [P, P, I64, I, P, I, P]),
            "oracle_embedding_4bit": (I, [P, P, I64, I64, I, I, P, I64, I, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments")


def _as_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    want = np.float32 if dtype == "f32" else np.uint16
    x = np.ascontiguousarray(x)
    if x.dtype != want:
        raise TypeError(f"{dtype} data must be passed as {want.__name__}, got {x.dtype}")
    return x


def code_table(qtype: str) -> np.ndarray:
    out = np.zeros(16, np.float32)
    _check(lib().oracle_code_table(QTYPES[qtype], _ptr(out)), "code_table")
    return out


def to_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    x = _as_storage(x, dtype)
    out = np.empty(x.size, np.float32)
    _check(lib().oracle_to_f32_array(_ptr(x), DTYPES[dtype], x.size, _ptr(out)), "to_f32")
    return out.reshape(x.shape)


def from_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.size, np.float32 if dtype == "f32" else np.uint16)
    _check(lib().oracle_from_f32_array(_ptr(x), x.size, DTYPES[dtype], _ptr(out)), "from_f32")
    return out.reshape(x.shape)


def quantize(x: np.ndarray, dtype: str, blocksize: int, qtype: str):
    """Returns (packed uint8[ceil(n/2)], absmax float32[ceil(n/blocksize)])."""
    x = _as_storage(x, dtype).reshape(-1)
    if blocksize <= 0:
        raise ValueError("blocksize must be positive")
    n = x.size
    packed = np.zeros((n + 1) // 2, np.uint8)
    absmax = np.zeros((n + blocksize - 1) // blocksize, np.float32)
    _check(lib().oracle_quantize(_ptr(x), DTYPES[dtype], n, blocksize, QTYPES[qtype],
                                 _ptr(packed), _ptr(absmax)), "quantize")
    return packed, absmax


def dequantize(packed: np.ndarray, absmax: np.ndarray, n: int, blocksize: int,
               qtype: str, out_dtype: str) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    absmax = np.ascontiguousarray(absmax, np.float32)
    assert packed.size >= (n + 1) // 2 and absmax.size >= (n + blocksize - 1) // blocksize
    out = np.empty(n, np.float32 if out_dtype == "f32" else np.uint16)
    _check(lib().oracle_dequantize(_ptr(packed), _ptr(absmax), n, blocksize, QTYPES[qtype],
                                   DTYPES[out_dtype], _ptr(out)), "dequantize")
    return out


def _weight_args(packed, absmax, N, K, blocksize):
    packed = np.ascontiguousarray(packed, np.uint8).reshape(-1)
    absmax = np.ascontiguousarray(absmax, np.float32).reshape(-1)
    assert packed.size >= (N * K + 1) // 2
    assert absmax.size >= (N * K + blocksize - 1) // blocksize
    return packed, absmax


def matmul(X, x_dtype, packed, absmax, bias, M, N, K, blocksize, qtype) -> np.ndarray:
    """float64 Y[M, N] = X @ dequant(W)^T (+ bias)."""
    X = _as_storage(X, x_dtype).reshape(-1)
    assert X.size == M * K
    packed, absmax = _weight_args(packed, absmax, N, K, blocksize)
    b = None if bias is None else _as_storage(bias, x_dtype).reshape(-1)
    Y = np.empty((M, N), np.float64)
    _check(lib().oracle_matmul(_ptr(X), DTYPES[x_dtype], _ptr(packed), _ptr(absmax), _ptr(b),
                               M, N, K, blocksize, QTYPES[qtype], _ptr(Y)), "matmul")
    return Y


def matmul_entries(X, x_dtype, packed, absmax, bias, M, N, K, blocksize, qtype, ms, js):
    X = _as_storage(X, x_dtype).reshape(-1)
    assert X.size == M * K
    packed, absmax = _weight_args(packed, absmax, N, K, blocksize)
    b = None if bias is None else _as_storage(bias, x_dtype).reshape(-1)
    ms = np.ascontiguousarray(ms, np.int64)
    js = np.ascontiguousarray(js, np.int64)
    Y = np.empty(ms.size, np.float64)
    _check(lib().oracle_matmul_entries(_ptr(X), DTYPES[x_dtype], _ptr(packed), _ptr(absmax),
                                       _ptr(b), M, N, K, blocksize, QTYPES[qtype], _ptr(ms),
                                       _ptr(js), ms.size, _ptr(Y)), "matmul_entries")
    return Y


def matmul_backward(dY, dy_dtype, packed, absmax, M, N, K, blocksize, qtype) -> np.ndarray:
    """float64 dX[M, K] = dY @ dequant(W)."""
    dY = _as_storage(dY, dy_dtype).reshape(-1)
    assert dY.size == M * N
    packed, absmax = _weight_args(packed, absmax, N, K, blocksize)
    dX = np.empty((M, K), np.float64)
    _check(lib().oracle_matmul_backward(_ptr(dY), DTYPES[dy_dtype], _ptr(packed), _ptr(absmax),
                                        M, N, K, blocksize, QTYPES[qtype], _ptr(dX)),
           "matmul_backward")
    return dX


def matmul_backward_entries(dY, dy_dtype, packed, absmax, M, N, K, blocksize, qtype, ms, ks):
    dY = _as_storage(dY, dy_dtype).reshape(-1)
    assert dY.size == M * N
    packed, absmax = _weight_args(packed, absmax, N, K, blocksize)
    ms = np.ascontiguousarray(ms, np.int64)
    ks = np.ascontiguousarray(ks, np.int64)
    dX = np.empty(ms.size, np.float64)
    _check(lib().oracle_matmul_backward_entries(_ptr(dY), DTYPES[dy_dtype], _ptr(packed),
                                                _ptr(absmax), M, N, K, blocksize,
                                                QTYPES[qtype], _ptr(ms), _ptr(ks), ms.size,
                                                _ptr(dX)), "matmul_backward_entries")
    return dX


def double_quant(absmax, group=256):
    """R9: (q uint8 [n], scales float32 [ceil(n / group)]) of an fp32 absmax array."""
    absmax = np.ascontiguousarray(absmax, np.float32).reshape(-1)
    if group < 1:
        raise ValueError("group must be >= 1")
    q = np.empty(absmax.size, np.uint8)
    scales = np.empty((absmax.size + group - 1) // group, np.float32)
    _check(lib().oracle_double_quant(_ptr(absmax), absmax.size, group, _ptr(q), _ptr(scales)),
           "double_quant")
    return q, scales


def dequant_absmax(q, scales, group=256):
    """R9 inverse: fp32(q) * fp32(scale / 255)."""
    q = np.ascontiguousarray(q, np.uint8).reshape(-1)
    scales = np.ascontiguousarray(scales, np.float32).reshape(-1)
    if group < 1 or scales.size != (q.size + group - 1) // group:
        raise ValueError("scales must hold one value per group")
    out = np.empty(q.size, np.float32)
    _check(lib().oracle_dequant_absmax(_ptr(q), _ptr(scales), q.size, group, _ptr(out)),
           "dequant_absmax")
    return out


def _code8(code) -> np.ndarray:
    code = np.ascontiguousarray(code, np.float32).reshape(-1)
    if code.size != 256:
        raise ValueError("an 8-bit code table has 256 entries")
    return code


def quantize_8bit(x: np.ndarray, dtype: str, blocksize: int, code) -> tuple:
    """R10: (q uint8[n], absmax float32[ceil(n/blocksize)]) against a 256-entry table."""
    x = _as_storage(x, dtype).reshape(-1)
    code = _code8(code)
    if blocksize <= 0:
        raise ValueError("blocksize must be positive")
    q = np.zeros(x.size, np.uint8)
    absmax = np.zeros((x.size + blocksize - 1) // blocksize, np.float32)
    _check(lib().oracle_quantize_8bit(_ptr(x), DTYPES[dtype], x.size, blocksize, _ptr(code),
                                      _ptr(q), _ptr(absmax)), "quantize_8bit")
    return q, absmax


def dequantize_8bit(q: np.ndarray, absmax: np.ndarray, n: int, blocksize: int, code,
                    out_dtype: str) -> np.ndarray:
    """R10 inverse: out[i] = RN_out(fp32(code[q[i]] * absmax[i // blocksize]))."""
    q = np.ascontiguousarray(q, np.uint8).reshape(-1)
    absmax = np.ascontiguousarray(absmax, np.float32).reshape(-1)
    code = _code8(code)
    assert q.size >= n and absmax.size >= (n + blocksize - 1) // blocksize
    out = np.empty(n, np.float32 if out_dtype == "f32" else np.uint16)
    _check(lib().oracle_dequantize_8bit(_ptr(q), _ptr(absmax), n, blocksize, _ptr(code),
                                        DTYPES[out_dtype], _ptr(out)), "dequantize_8bit")
    return out


def embedding_4bit(packed: np.ndarray, absmax: np.ndarray, V: int, D: int, blocksize: int,
                   qtype: str, idx, out_dtype: str) -> np.ndarray:
    """R11: rows idx of a [V, D] table quantized as one flat array -> [len(idx), D]."""
    packed = np.ascontiguousarray(packed, np.uint8).reshape(-1)
    absmax = np.ascontiguousarray(absmax, np.float32).reshape(-1)
    idx = np.ascontiguousarray(idx, np.int64).reshape(-1)
    assert packed.size >= (V * D + 1) // 2 and absmax.size >= (V * D + blocksize - 1) // blocksize
    out = np.empty(idx.size * D, np.float32 if out_dtype == "f32" else np.uint16)
    _check(lib().oracle_embedding_4bit(_ptr(packed), _ptr(absmax), V, D, blocksize, QTYPES[qtype],
                                       _ptr(idx), idx.size, DTYPES[out_dtype], _ptr(out)),
           "embedding_4bit")
    return out.reshape(idx.size, D)
