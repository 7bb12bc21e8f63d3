"""Large-batch apply of an unstructured (CSR) S on the tensor cores, against
the float64 oracle: each 64-column block of S is decompressed into shared
memory for the dense MMA, then U·Zᵀ joins the same accumulator.  Batches of
65 tokens or more take this path for bf16 CSR layers (n % 8 == 0) whose rows
have strictly ascending columns; otherwise the CUDA-core decode kernel runs."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth
from sparse_rank_linear_03_b200.configs import ATTN4096, STACK7B

from gpu_util import check_close, csr_dense_rows, dev, factors, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def f64(b):
    return oracle.bits_to_f64(b, "bf16")


def build(hsl, m, n, r, frac, seed, split_dtype="bf16", stand_in=False):
    Wf = synth.student_t_f32(m, n, seed)
    W = synth.as_storage(Wf, split_dtype)
    L = hsl.Layer(m, n, r, "csr", "bf16")
    L.split(dev(W, split_dtype), frac, None)
    ref = oracle.split_topk(W, frac, split_dtype)
    vals = ref["val"] if split_dtype == "bf16" else oracle.f32_to_bf16_bits(ref["val"].view(np.float32))
    if stand_in:
        Uf, Vf = synth.stand_in_factors(m, n, r, seed + 2)
        U, V = synth.to_bf16_bits(Uf), synth.to_bf16_bits(Vf)
    else:
        U, V = factors(oracle.bits_to_f64(ref["R"], split_dtype), r, "bf16", seed)
    L.pack(dev(U, "bf16"), dev(V, "bf16"))
    return L, ref["row_ptr"], ref["col"], vals, U, V


def ref_rows(rp, col, vals, U, V, X, rows, n):
    S = csr_dense_rows(rp, col, f64(vals), rows, n)
    return oracle.apply_rows(np.arange(len(rows)), S, f64(U[rows]), f64(V), f64(X))


@pytest.mark.parametrize("m,n,r,T,frac", [
    (300, 128, 8, 100, 0.05), (129, 72, 0, 300, 0.1), (1000, 4096, 128, 65, 0.02),
    (513, 1000, 16, 257, 0.03), (64, 64, 256, 70, 0.5), (257, 8, 3, 513, 0.3),
])
def test_csr_prefill_small_shapes(hsl, m, n, r, T, frac):
    L, rp, col, vals, U, V = build(hsl, m, n, r, frac, m + n + r)
    X = synth.to_bf16_bits(synth.normal_f32(T, n, T))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    check_close(f64(host(Y)), ref_rows(rp, col, vals, U, V, X, np.arange(m), n), "bf16")


def test_csr_prefill_attn4096_2048_tokens(hsl):
    lay = ATTN4096.layers[0]
    L, rp, col, vals, U, V = build(hsl, lay.m, lay.n, ATTN4096.r, ATTN4096.frac, lay.seed,
                                   split_dtype="f32", stand_in=True)
    X = synth.to_bf16_bits(synth.normal_f32(2048, lay.n, lay.seed + 1))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    rows = np.sort(np.random.default_rng(6).choice(lay.m, 384, replace=False))
    rows[-1] = lay.m - 1
    check_close(f64(host(Y))[:, rows], ref_rows(rp, col, vals, U, V, X, rows, lay.n), "bf16")


def test_csr_prefill_7b_down_projection(hsl):
    """The 4096×11008 down projection at 3 %, r = 128, 1024 tokens."""
    lay = STACK7B.layers[6]
    L, rp, col, vals, U, V = build(hsl, lay.m, lay.n, STACK7B.r, STACK7B.frac, lay.seed,
                                   split_dtype="f32", stand_in=True)
    X = synth.to_bf16_bits(synth.normal_f32(1024, lay.n, lay.seed + 1))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    rows = np.sort(np.random.default_rng(7).choice(lay.m, 256, replace=False))
    check_close(f64(host(Y))[:, rows], ref_rows(rp, col, vals, U, V, X, rows, lay.n), "bf16")


def test_csr_prefill_matches_the_decode_kernel(hsl):
    """One layer, 128 tokens: the tensor-core path in one call and the CUDA-core
    path in calls of 8 tokens agree to bf16 output rounding."""
    L, *_ = build(hsl, 700, 512, 24, 0.04, 9)
    X = dev(synth.to_bf16_bits(synth.normal_f32(128, 512, 3)), "bf16")
    Yp = L.apply(X)
    Yd = torch.cat([L.apply(X[i:i + 8].contiguous()) for i in range(0, 128, 8)])
    assert oracle.rel_err(f64(host(Yp)), f64(host(Yd))) <= 2e-2


def test_imported_rows_out_of_order_take_the_decode_path(hsl):
    """An imported S whose row lists a column twice (the oracle adds both) is
    applied by the decode kernel, which sums every entry."""
    m, n = 96, 64
    rng = np.random.default_rng(4)
    rp = np.arange(0, 3 * m + 1, 3, dtype=np.int32)
    col = np.sort(rng.integers(0, n, size=(m, 3)), axis=1).astype(np.int32)
    col[:, 1] = col[:, 0]                      # a repeated column in every row
    vals = synth.to_bf16_bits(rng.standard_normal(3 * m).astype(np.float32))
    L = hsl.Layer(m, n, 0, "csr", "bf16")
    L.set_sparse_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(col.reshape(-1)).cuda(),
                     dev(vals, "bf16"))
    L.pack(None, None)
    X = synth.to_bf16_bits(synth.normal_f32(100, n, 5))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    S = oracle.csr_to_dense(m, n, rp, col.reshape(-1), f64(vals))
    check_close(f64(host(Y)), oracle.apply(S, f64(X)), "bf16")
