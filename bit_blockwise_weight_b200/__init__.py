"""Python binding of libbnb4.so: 4-bit blockwise weight quantization on B200.

Two layers, both argument marshalling only (every step of the computation
runs in the library's CUDA kernels):

* ``bnb4_quantize``, ``bnb4_dequantize``, ``bnb4_gemv``, ``bnb4_gemm``,
  ``bnb4_gemm_backward``, ``bnb4_gemv_dq``, ``bnb4_gemm_dq``, ``bnb4_gemm_backward_dq``,
  ``bnb4_double_quant``, ``bnb4_dequant_absmax``,
  ``bnb4_quantize_8bit``, ``bnb4_dequantize_8bit``, ``bnb4_embedding_4bit``,
  ``bnb4_device_status``, ``bnb4_selftest_wait_timeout``: the C ABI of
  ``include/bnb4.h`` one to one (raw
  device pointers as ints, sizes, enums, a ``cudaStream_t`` as an int).
  They return the integer status.
* ``quantize_4bit``, ``dequantize_4bit``, ``gemv_4bit``, ``gemm_4bit``,
  ``gemm_4bit_backward``, ``double_quant``, ``dequant_absmax``,
  ``gemv_4bit_dq``, ``gemm_4bit_dq``, ``gemm_4bit_backward_dq``, ``quantize_8bit``, ``dequantize_8bit``,
  ``embedding_4bit``, ``device_status``: take torch CUDA tensors (the 8-bit
  code table on the host), allocate outputs with torch, call the C ABI on the
  current stream and raise ``Bnb4Error`` on a non-OK status.

Importing the package loads the shared library and fails loudly if it is
missing.  There is no CPU or pure-PyTorch fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbnb4.so")

NF4, FP4 = 0, 1
F32, F16, BF16 = 0, 1, 2
QTYPES = {"nf4": NF4, "fp4": FP4}
STATUS_OK = 0


class Bnb4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libbnb4.so not found at {LIB_PATH}; build it with "
            "`python bit_blockwise_weight_b200/build.py` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sigs = {
        "bnb4_version": (I, []),
        "bnb4_status_string": (ctypes.c_char_p, [I]),
        "bnb4_quantize": (I, [P, P, P, I64, I, I, I, P]),
        "bnb4_dequantize": (I, [P, P, P, I64, I, I, I, P]),
        "bnb4_gemv": (I, [P, P, P, P, P, I64, I64, I, I, I, P]),
        "bnb4_gemm": (I, [P, P, P, P, P, I64, I64, I64, I, I, I, P]),
        "bnb4_gemm_backward": (I, [P, P, P, P, I64, I64, I64, I, I, I, P]),
        "bnb4_gemv_dq": (I, [P, P, P, P, I, P, P, I64, I64, I, I, I, P]),
        "bnb4_gemm_dq": (I, [P, P, P, P, I, P, P, I64, I64, I64, I, I, I, P]),
        "bnb4_gemm_backward_dq": (I, [P, P, P, P, I, P, I64, I64, I64, I, I, I, P]),
        "bnb4_quantize_8bit": (I, [P, P, P, I64, I, P, I, P]),
        "bnb4_dequantize_8bit": (I, [P, P, P, I64, I, P, I, P]),
        "bnb4_embedding_4bit": (I, [P, P, I64, I64, I, I, P, I64, P, I, P]),
        "bnb4_double_quant": (I, [P, I64, I, P, P, P]),
        "bnb4_dequant_absmax": (I, [P, P, I64, I, P, P]),
        "bnb4_device_status": (I, [P]),
        "bnb4_selftest_wait_timeout": (I, [P]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


_lib = _load()

# ------------------------------------------------------------------ C ABI

bnb4_version = _lib.bnb4_version
bnb4_quantize = _lib.bnb4_quantize
bnb4_dequantize = _lib.bnb4_dequantize
bnb4_gemv = _lib.bnb4_gemv
bnb4_gemm = _lib.bnb4_gemm
bnb4_gemm_backward = _lib.bnb4_gemm_backward
bnb4_gemv_dq = _lib.bnb4_gemv_dq
bnb4_gemm_dq = _lib.bnb4_gemm_dq
bnb4_gemm_backward_dq = _lib.bnb4_gemm_backward_dq
bnb4_quantize_8bit = _lib.bnb4_quantize_8bit
bnb4_dequantize_8bit = _lib.bnb4_dequantize_8bit
bnb4_embedding_4bit = _lib.bnb4_embedding_4bit
bnb4_double_quant = _lib.bnb4_double_quant
bnb4_dequant_absmax = _lib.bnb4_dequant_absmax
bnb4_device_status = _lib.bnb4_device_status
bnb4_selftest_wait_timeout = _lib.bnb4_selftest_wait_timeout


def status_string(status: int) -> str:
    return _lib.bnb4_status_string(int(status)).decode()


def library_path() -> str:
    return LIB_PATH


# ------------------------------------------------------- torch-level wrappers

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    codes = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _qtype(q) -> int:
    return QTYPES[q] if isinstance(q, str) else int(q)


def _stream(stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check(status: int, what: str):
    if status != STATUS_OK:
        raise Bnb4Error(status, what)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def quantize_4bit(x, blocksize: int = 64, quant_type="nf4", stream=None):
    """x: any-shape f32/f16/bf16 CUDA tensor -> (packed uint8[ceil(n/2)], absmax f32[ceil(n/B)])."""
    torch = _torch()
    _need_cuda(x)
    n = x.numel()
    packed = torch.empty((n + 1) // 2, dtype=torch.uint8, device=x.device)
    absmax = torch.empty((n + blocksize - 1) // blocksize, dtype=torch.float32, device=x.device)
    _check(bnb4_quantize(_ptr(x), _ptr(packed), _ptr(absmax), n, blocksize, _qtype(quant_type),
                         _dtype_code(x), _stream(stream)), "bnb4_quantize")
    return packed, absmax


def quantize_4bit_into(x, packed, absmax, blocksize: int = 64, quant_type="nf4", stream=None):
    """quantize_4bit into caller-provided outputs (no allocation)."""
    _need_cuda(x, packed, absmax)
    _check(bnb4_quantize(_ptr(x), _ptr(packed), _ptr(absmax), x.numel(), blocksize,
                         _qtype(quant_type), _dtype_code(x), _stream(stream)), "bnb4_quantize")
    return packed, absmax


def dequantize_4bit(packed, absmax, n: int, blocksize: int = 64, quant_type="nf4",
                    dtype=None, out=None, stream=None):
    """-> out[n] of dtype (default bfloat16)."""
    torch = _torch()
    _need_cuda(packed, absmax)
    if out is None:
        out = torch.empty(n, dtype=dtype or torch.bfloat16, device=packed.device)
    _need_cuda(out)
    _check(bnb4_dequantize(_ptr(packed), _ptr(absmax), _ptr(out), n, blocksize,
                           _qtype(quant_type), _dtype_code(out), _stream(stream)),
           "bnb4_dequantize")
    return out


def gemv_4bit(x, packed, absmax, N: int, K: int, bias=None, blocksize: int = 64,
              quant_type="nf4", out=None, stream=None):
    """x [K] -> y [N] = x @ dequant(W)^T (+ bias)."""
    torch = _torch()
    _need_cuda(x, packed, absmax, bias)
    y = out if out is not None else torch.empty(N, dtype=x.dtype, device=x.device)
    _check(bnb4_gemv(_ptr(x), _ptr(packed), _ptr(absmax), _ptr(bias), _ptr(y), N, K, blocksize,
                     _qtype(quant_type), _dtype_code(x), _stream(stream)), "bnb4_gemv")
    return y


def gemv_4bit_dq(x, packed, absmax_q, absmax_scales, N: int, K: int, bias=None,
                 blocksize: int = 64, quant_type="nf4", group: int = 256, out=None, stream=None):
    """gemv_4bit with the absmax given as double_quant's (codes, scales)."""
    torch = _torch()
    _need_cuda(x, packed, absmax_q, absmax_scales, bias)
    y = out if out is not None else torch.empty(N, dtype=x.dtype, device=x.device)
    _check(bnb4_gemv_dq(_ptr(x), _ptr(packed), _ptr(absmax_q), _ptr(absmax_scales), group, _ptr(bias),
                        _ptr(y), N, K, blocksize, _qtype(quant_type), _dtype_code(x), _stream(stream)),
           "bnb4_gemv_dq")
    return y


def gemm_4bit(X, packed, absmax, N: int, bias=None, blocksize: int = 64, quant_type="nf4",
              out=None, stream=None):
    """X [M, K] -> Y [M, N] = X @ dequant(W)^T (+ bias)."""
    torch = _torch()
    _need_cuda(X, packed, absmax, bias)
    M, K = X.shape
    Y = out if out is not None else torch.empty(M, N, dtype=X.dtype, device=X.device)
    _check(bnb4_gemm(_ptr(X), _ptr(packed), _ptr(absmax), _ptr(bias), _ptr(Y), M, N, K, blocksize,
                     _qtype(quant_type), _dtype_code(X), _stream(stream)), "bnb4_gemm")
    return Y


def gemm_4bit_backward(dY, packed, absmax, K: int, blocksize: int = 64, quant_type="nf4",
                       out=None, stream=None):
    """dY [M, N] -> dX [M, K] = dY @ dequant(W)."""
    torch = _torch()
    _need_cuda(dY, packed, absmax)
    M, N = dY.shape
    dX = out if out is not None else torch.empty(M, K, dtype=dY.dtype, device=dY.device)
    _check(bnb4_gemm_backward(_ptr(dY), _ptr(packed), _ptr(absmax), _ptr(dX), M, N, K, blocksize,
                              _qtype(quant_type), _dtype_code(dY), _stream(stream)),
           "bnb4_gemm_backward")
    return dX


def gemm_4bit_dq(X, packed, absmax_q, absmax_scales, N: int, bias=None, blocksize: int = 64,
                 quant_type="nf4", group: int = 256, out=None, stream=None):
    """gemm_4bit with the absmax given as double_quant's (codes, scales)."""
    torch = _torch()
    _need_cuda(X, packed, absmax_q, absmax_scales, bias)
    M, K = X.shape
    Y = out if out is not None else torch.empty(M, N, dtype=X.dtype, device=X.device)
    _check(bnb4_gemm_dq(_ptr(X), _ptr(packed), _ptr(absmax_q), _ptr(absmax_scales), group, _ptr(bias), _ptr(Y),
                        M, N, K, blocksize, _qtype(quant_type), _dtype_code(X), _stream(stream)), "bnb4_gemm_dq")
    return Y


def gemm_4bit_backward_dq(dY, packed, absmax_q, absmax_scales, K: int, blocksize: int = 64,
                          quant_type="nf4", group: int = 256, out=None, stream=None):
    """gemm_4bit_backward with the absmax given as double_quant's (codes, scales)."""
    torch = _torch()
    _need_cuda(dY, packed, absmax_q, absmax_scales)
    M, N = dY.shape
    dX = out if out is not None else torch.empty(M, K, dtype=dY.dtype, device=dY.device)
    _check(bnb4_gemm_backward_dq(_ptr(dY), _ptr(packed), _ptr(absmax_q), _ptr(absmax_scales), group, _ptr(dX),
                                 M, N, K, blocksize, _qtype(quant_type), _dtype_code(dY), _stream(stream)),
           "bnb4_gemm_backward_dq")
    return dX


def double_quant(absmax, group: int = 256, out=None, stream=None):
    """absmax float32 [n] (CUDA) -> (absmax_q uint8 [n], scales float32 [ceil(n/group)]);
    out = (absmax_q, scales) writes into caller-provided buffers."""
    torch = _torch()
    _need_cuda(absmax)
    if absmax.dtype != torch.float32:
        raise TypeError("absmax must be float32")
    n = absmax.numel()
    if out is not None:
        q, scales = out
        _need_cuda(q, scales)
        if q.numel() != n or scales.numel() != (n + group - 1) // group:
            raise ValueError("out buffers have the wrong sizes")
    else:
        q = torch.empty(n, dtype=torch.uint8, device=absmax.device)
        scales = torch.empty((n + group - 1) // group, dtype=torch.float32, device=absmax.device)
    _check(bnb4_double_quant(_ptr(absmax), n, group, _ptr(q), _ptr(scales), _stream(stream)),
           "bnb4_double_quant")
    return q, scales


def dequant_absmax(absmax_q, scales, group: int = 256, out=None, stream=None):
    """Inverse of double_quant -> absmax float32 [n]."""
    torch = _torch()
    _need_cuda(absmax_q, scales)
    n = absmax_q.numel()
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=absmax_q.device)
    _need_cuda(out)
    _check(bnb4_dequant_absmax(_ptr(absmax_q), _ptr(scales), n, group, _ptr(out), _stream(stream)),
           "bnb4_dequant_absmax")
    return out


def _host_code8(code):
    torch = _torch()
    c = torch.as_tensor(code, dtype=torch.float32).detach().to("cpu").contiguous().reshape(-1)
    if c.numel() != 256:
        raise ValueError("an 8-bit code table has 256 entries")
    return c  # kept alive by the caller for the duration of the call


def quantize_8bit(x, code, blocksize: int = 64, stream=None):
    """x: f32/f16/bf16 CUDA tensor; code: 256 ascending entries (host).
    -> (q uint8[n], absmax f32[ceil(n/B)])."""
    torch = _torch()
    _need_cuda(x)
    c = _host_code8(code)
    n = x.numel()
    q = torch.empty(n, dtype=torch.uint8, device=x.device)
    absmax = torch.empty((n + blocksize - 1) // blocksize, dtype=torch.float32, device=x.device)
    _check(bnb4_quantize_8bit(_ptr(x), _ptr(q), _ptr(absmax), n, blocksize, c.data_ptr(), _dtype_code(x),
                              _stream(stream)), "bnb4_quantize_8bit")
    return q, absmax


def dequantize_8bit(q, absmax, code, blocksize: int = 64, dtype=None, out=None, stream=None):
    """-> out[n] of dtype (default bfloat16)."""
    torch = _torch()
    _need_cuda(q, absmax)
    c = _host_code8(code)
    n = q.numel()
    if out is None:
        out = torch.empty(n, dtype=dtype or torch.bfloat16, device=q.device)
    _need_cuda(out)
    _check(bnb4_dequantize_8bit(_ptr(q), _ptr(absmax), _ptr(out), n, blocksize, c.data_ptr(), _dtype_code(out),
                                _stream(stream)), "bnb4_dequantize_8bit")
    return out


def embedding_4bit(packed, absmax, V: int, D: int, idx, blocksize: int = 64, quant_type="nf4",
                   dtype=None, out=None, stream=None):
    """Rows idx (int64 CUDA tensor) of a [V, D] table quantized by quantize_4bit -> [len(idx), D]."""
    torch = _torch()
    _need_cuda(packed, absmax, idx)
    if idx.dtype != torch.int64:
        raise TypeError("indices must be int64")
    n_idx = idx.numel()
    if out is None:
        out = torch.empty(n_idx, D, dtype=dtype or torch.bfloat16, device=packed.device)
    _need_cuda(out)
    _check(bnb4_embedding_4bit(_ptr(packed), _ptr(absmax), V, D, blocksize, _qtype(quant_type), _ptr(idx), n_idx,
                               _ptr(out), _dtype_code(out), _stream(stream)), "bnb4_embedding_4bit")
    return out


def device_status(stream=None) -> int:
    """Synchronise the stream, then read and clear the count of bounded device
    waits that gave up: STATUS_OK, or the BNB4_ERR_TIMEOUT / BNB4_ERR_CUDA code."""
    return int(bnb4_device_status(_stream(stream)))
