"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module draws random numbers and converts dtypes; it holds none of the
method's arithmetic (no split, no factorisation, no product).  Both the CUDA
path and the oracle consume exactly what it returns.

Recipe (stand-in for the LLM layers the pages talk about; no real weights or
evaluation data are used):

* W = 0.02 · t₃ (Student-t, ν = 3) drawn in float64 with
  ``numpy.random.default_rng(seed).standard_t(3, size=(m, n))``, rounded to
  float32 (round-to-nearest-even).  Heavy-tailed as the pages assume for LLM
  weights.  bf16 layers round that float32 once more to bfloat16 (RNE).
* X ~ N(0, 1) from ``default_rng(seed + 1).standard_normal((B, n))``, rounded
  to the layer's dtype.
* The 224-matrix 7B stack in the bench draws W on the device instead
  (:func:`student_t_device`, torch's seeded CUDA generator: t₃ = N / √(χ²₃/3)
  with χ²₃ the sum of three squared normals), because drawing its 6.5 G
  entries on the host takes minutes; it is the same distribution.
* Bench-side stand-in factors: U, V with i.i.d. N(0, s²) entries from
  ``default_rng(seed + 2)`` (s chosen so that (U Vᵀ)ᵢⱼ has standard deviation
  about 0.01).  Throughput does not depend on the factor values; the tests use
  the oracle's truncated SVD of the residual instead.
"""
from __future__ import annotations

import numpy as np
import torch


def student_t_f32(m: int, n: int, seed: int, scale: float = 0.02, df: float = 3.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (scale * rng.standard_t(df, size=(m, n))).astype(np.float32)


def skew_columns(W: np.ndarray, seed: int, frac: float = 0.01, factor: float = 8.0) -> np.ndarray:
    """Labelled variant: scale a random 1 % of input columns by 8 (outlier channels)."""
    rng = np.random.default_rng(seed + 7)
    n = W.shape[1]
    cols = rng.choice(n, size=max(1, int(frac * n)), replace=False)
    out = W.copy()
    out[:, cols] *= np.float32(factor)
    return out


def normal_f32(b: int, n: int, seed: int) -> np.ndarray:
    return np.random.default_rng(seed).standard_normal((b, n)).astype(np.float32)


def stand_in_factors(m: int, n: int, r: int, seed: int, target_std: float = 0.01):
    """Gaussian U [m, r], V [n, r] in float32 for throughput runs."""
    rng = np.random.default_rng(seed)
    s = (target_std ** 2 / max(r, 1)) ** 0.25 if r else 0.0
    U = (s * rng.standard_normal((m, r))).astype(np.float32)
    V = (s * rng.standard_normal((n, r))).astype(np.float32)
    return U, V


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 → bfloat16 (RNE, torch's CPU conversion) as uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def as_storage(x_f32: np.ndarray, dtype: str) -> np.ndarray:
    """The storage bits of a float32 array in ``dtype`` ("f32" or "bf16")."""
    if dtype == "f32":
        return np.ascontiguousarray(x_f32, dtype=np.float32)
    if dtype == "bf16":
        return to_bf16_bits(x_f32)
    raise ValueError(dtype)


def torch_from_storage(bits: np.ndarray, dtype: str, device="cpu") -> torch.Tensor:
    """Wrap storage bits as a torch tensor of the matching dtype."""
    if dtype == "f32":
        a = np.ascontiguousarray(bits)
        # uint32 storage bits are reinterpreted, float arrays taken as values
        a = a.view(np.float32) if a.dtype in (np.uint32, np.int32) else a.astype(np.float32, copy=False)
        t = torch.from_numpy(a)
    else:
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def storage_from_torch(t: torch.Tensor) -> np.ndarray:
    """Inverse of :func:`torch_from_storage` (copies to host)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy().copy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def student_t_device(m: int, n: int, seed: int, device, scale: float = 0.02) -> torch.Tensor:
    """0.02 · t₃ as float32 on `device`, from torch's seeded generator there."""
    g = torch.Generator(device=device).manual_seed(seed)
    z = torch.randn(m, n, generator=g, device=device)
    chi2 = torch.zeros(m, n, device=device)
    for _ in range(3):
        chi2.add_(torch.randn(m, n, generator=g, device=device).square_())
    return (scale * z * torch.rsqrt(chi2 / 3.0)).contiguous()


def stand_in_factors_device(m: int, n: int, r: int, seed: int, device, dtype=torch.bfloat16,
                            target_std: float = 0.01):
    """Device twin of :func:`stand_in_factors` (same scale, torch's generator)."""
    g = torch.Generator(device=device).manual_seed(seed)
    s = (target_std ** 2 / max(r, 1)) ** 0.25 if r else 0.0
    U = (s * torch.randn(m, r, generator=g, device=device)).to(dtype)
    V = (s * torch.randn(n, r, generator=g, device=device)).to(dtype)
    return U.contiguous(), V.contiguous()
