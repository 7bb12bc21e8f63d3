"""Helpers shared by the GPU parity tests (inputs, conversions, oracle calls)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_rank_linear_03_b200 import synth

TOL = {"f32": 1e-5, "bf16": 1e-2}
# Element-wise relative error (denominator max(|y*|, 1e-3·max|y*|)), reported
# beside the normwise one.  bf16: the output rounding alone is 2^-9 per element,
# so the normwise bound 1e-2 holds element-wise too.  f32: an output that nearly
# cancels carries the fp32 accumulation error of its terms (~1e-7 of the row
# maximum) over a denominator of 1e-3 of it, so the element-wise bound is 1e-3.
ELEM_TOL = {"f32": 1e-3, "bf16": 1e-2}


def check_close(Y64: np.ndarray, Yref: np.ndarray, dtype: str) -> tuple[float, float]:
    """Both error measures of the oracle against their bounds; returns them."""
    e = oracle.rel_err(Y64, Yref)
    el = oracle.elem_rel_err(Y64, Yref)
    assert e <= TOL[dtype], f"normwise {e:.3e} > {TOL[dtype]}"
    assert el <= ELEM_TOL[dtype], f"element-wise {el:.3e} > {ELEM_TOL[dtype]}"
    return e, el


def dev(bits: np.ndarray, dtype: str) -> torch.Tensor:
    return synth.torch_from_storage(bits, dtype, "cuda")


def host(t: torch.Tensor) -> np.ndarray:
    return synth.storage_from_torch(t)


def factors(R64: np.ndarray, r: int, dtype: str, seed: int = 0, exact: bool = False):
    """Oracle low-rank factors of the residual, rounded to the layer dtype.

    Returns (U_bits, V_bits) — what both sides consume."""
    if r == 0:
        m, n = R64.shape
        return (synth.as_storage(np.zeros((m, 0), np.float32), dtype),
                synth.as_storage(np.zeros((n, 0), np.float32), dtype))
    if exact or min(R64.shape) <= 1100:
        U, V = oracle.lowrank_svd(R64, r)
    else:
        omega = np.random.default_rng(seed + 99).standard_normal((R64.shape[1], r + 10))
        U, V = oracle.lowrank_randomized(R64, r, omega, power_iters=1)
    return (synth.as_storage(U.astype(np.float32), dtype),
            synth.as_storage(V.astype(np.float32), dtype))


def csr_dense_rows(rp, col, val64, rows, n):
    out = np.zeros((len(rows), n))
    for t, i in enumerate(rows):
        a, b = rp[i], rp[i + 1]
        out[t, col[a:b]] = val64[a:b]
    return out


def nm24_dense_rows(val64, idx, rows):
    return oracle.nm24_to_dense(val64[rows], idx[rows])


def as_bits(a: np.ndarray) -> np.ndarray:
    """Storage bits of an f32/bf16 array (so that -0.0 != +0.0 in comparisons)."""
    return a.view(np.uint32) if a.dtype == np.float32 else a


def check_csr_equal(got: dict, ref: dict, dtype_val: str):
    rp = got["row_ptr"].cpu().numpy()
    assert np.array_equal(rp, ref["row_ptr"]), "row_ptr differs"
    assert np.array_equal(got["col"].cpu().numpy(), ref["col"]), "col differs"
    assert np.array_equal(as_bits(host(got["val"])), as_bits(ref["val"])), "values differ"


def ref_values(vals_bits: np.ndarray, w_dtype: str, layer_dtype: str) -> np.ndarray:
    """The kept values as the layer stores them (f32 → bf16 RNE; bf16 → f32 exact)."""
    if w_dtype == layer_dtype:
        return vals_bits
    if layer_dtype == "bf16":
        return oracle.f32_to_bf16_bits(vals_bits.view(np.float32))
    return oracle.bits_to_f64(vals_bits, "bf16").astype(np.float32)
