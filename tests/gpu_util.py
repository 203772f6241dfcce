"""Helpers for the GPU parity tests: move seeded inputs between numpy storage and CUDA tensors."""
import numpy as np
import torch

TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
# relative L2 bound for the 4-bit matmuls (bf16/fp16 out, fp32 accumulate) against the
# float64 product of the dequantized weights
MATMUL_TOL = 5e-3


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if dtype == "f32":
        return torch.from_numpy(a.astype(np.float32, copy=False)).cuda()
    t = torch.from_numpy(a.view(np.int16)).cuda()
    return t.view(TORCH[dtype])


def to_host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def as_f64(storage: np.ndarray, dtype: str) -> np.ndarray:
    import oracle
    return oracle.to_f32(storage, dtype).astype(np.float64)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, np.float64).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def unpack_nibbles(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.size * 2, np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 15
    return out[:n]


# Unit roundoff of the 16-bit compute dtypes: bf16 has an 8-bit significand,
# fp16 an 11-bit one, so rounding to them moves a value by at most 2^-8 / 2^-11
# of itself.
UNIT_ROUNDOFF = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11}


def elementwise_excess(got, ref, absdot, dt, K):
    """How far the worst output lies outside its own error bound (<= 0: every
    output inside).  The 16-bit matmuls meet the weight rounded once to the
    compute dtype (RN_dt(code) * absmax, or RN_dt(code * absmax)), multiply it
    exactly by x in fp32, sum in fp32 and round the result once to the dtype:
        |y - y_ref| <= u_dt (sum_k |x_k w_k| + |b|) + u_dt |y_ref|
                       + (K + 4) 2^-24 (sum_k |x_k w_k| + |b|)
    with a 1 % margin and an absolute floor at the smallest fp16 subnormal.
    absdot is sum_k |x_k w_k| + |b| per output.  A localised mistake (one
    block's scale, one column) breaks this bound long before it moves the
    relative L2 over the whole tensor."""
    u = UNIT_ROUNDOFF[dt]
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    absdot = np.asarray(absdot, np.float64)
    tol = 1.01 * (u * absdot + u * np.abs(ref)) + (K + 4) * 2.0 ** -24 * absdot + 2.0 ** -24
    return float(np.max(np.abs(got - ref) - tol))
