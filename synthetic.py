"""Seeded synthetic inputs shaped like the LLM workloads of the 4-bit path.

This module only draws random numbers.  It holds none of the quantization or
matmul arithmetic, so the CUDA path and the CPU oracle can both take their
inputs from it.

Recipe (the pages fix no distribution beyond "normally distributed" LLM
weights, "mps-bitsandbytes 0.4.7", Features table, NF4 row):
  * ``torch.Generator('cpu').manual_seed(seed)``;
  * ``torch.randn(shape, dtype=float32) * sigma``;
  * optional outliers: ``mask = torch.rand(n) < frac`` drawn after the normal
    draw, then ``x[mask] *= scale``;
  * a cast to the target dtype with torch's round-to-nearest-even.
"""
from __future__ import annotations

import torch

TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def normal(shape, seed: int, sigma: float = 1.0, dtype: str = "f32",
           outlier_frac: float = 0.0, outlier_scale: float = 20.0,
           device: str = "cpu") -> torch.Tensor:
    """A tensor of the given shape and dtype, drawn as described above.

    The generator lives on `device`; CPU and CUDA generators give different
    (each reproducible) streams, so inputs that the CPU oracle must see are
    drawn on the CPU.
    """
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if sigma != 1.0:
        x.mul_(sigma)
    if outlier_frac > 0.0:
        mask = torch.rand(x.numel(), generator=g, device=device) < outlier_frac
        x.view(-1)[mask] *= outlier_scale
    return x.to(TORCH_DTYPES[dtype])


def weight(N: int, K: int, seed: int = 0, sigma: float = 0.02) -> torch.Tensor:
    """fp32 weight [N, K] (out x in, row-major like nn.Linear.weight)."""
    return normal((N, K), seed, sigma, "f32")


def activations(M: int, K: int, seed: int = 1, dtype: str = "bf16") -> torch.Tensor:
    return normal((M, K), seed, 1.0, dtype)


def bias(N: int, seed: int = 2, dtype: str = "bf16") -> torch.Tensor:
    return normal((N,), seed, 1.0, dtype)


def grad_output(M: int, N: int, seed: int = 3, dtype: str = "bf16") -> torch.Tensor:
    return normal((M, N), seed, 1.0, dtype)


def roundtrip_tensor(n: int, seed: int, dtype: str, device: str = "cpu") -> torch.Tensor:
    """1-D N(0, 1) tensor with 1% of the entries scaled by 20 (outliers)."""
    return normal((n,), seed, 1.0, dtype, outlier_frac=0.01, outlier_scale=20.0, device=device)


def absmax_values(n: int, seed: int = 4, sigma: float = 0.02, zero_frac: float = 0.0) -> torch.Tensor:
    """n positive fp32 values shaped like the block maxima of N(0, sigma) weights
    (about 2.4 sigma for blocks of 64, a narrow spread): sigma * 2.4 *
    exp(0.15 * randn).  With zero_frac > 0, a ``torch.rand(n) < zero_frac``
    mask drawn after that sets values to 0 (all-zero blocks)."""
    g = torch.Generator("cpu").manual_seed(seed)
    a = torch.exp(torch.randn(n, generator=g, dtype=torch.float32) * 0.15) * (2.4 * sigma)
    if zero_frac > 0.0:
        a[torch.rand(n, generator=g) < zero_frac] = 0.0
    return a


def storage_numpy(t: torch.Tensor):
    """Raw storage as numpy: float32 stays float32, 16-bit types become uint16 bits."""
    t = t.contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy()
    return t.view(torch.int16).numpy().view("uint16")
