"""Parity of the tensor-core (large-batch) 2:4 apply with the float64 oracle.

Batches of 16 tokens or more on bf16 2:4 layers with n % 64 == 0 take the
tcgen05 path: Z = X·V, then S·Xᵀ + U·Zᵀ in one TMEM accumulator.  Z is rounded
to bf16 before the second product, well inside the 1e-2 bound."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth
from sparse_rank_linear_03_b200.configs import MLP70B, MLP_UP_11008

from gpu_util import TOL, check_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def f64(b):
    return oracle.bits_to_f64(b, "bf16")


def build(hsl, m, n, r, seed, stand_in=False):
    W = synth.to_bf16_bits(synth.student_t_f32(m, n, seed))
    L = hsl.Layer(m, n, r, "nm24", "bf16")
    L.split(dev(W, "bf16"), 0.5, None)
    if stand_in:
        Uf, Vf = synth.stand_in_factors(m, n, r, seed + 2)
    else:
        ref = oracle.split_24(W, "bf16")
        Ud, Vd = oracle.lowrank_svd(f64(ref["R"]), r) if r else (np.zeros((m, 0)), np.zeros((n, 0)))
        Uf, Vf = Ud.astype(np.float32), Vd.astype(np.float32)
    U, V = synth.to_bf16_bits(Uf), synth.to_bf16_bits(Vf)
    L.pack(dev(U, "bf16"), dev(V, "bf16"))
    return L, W, U, V


def ref_rows(W, U, V, X, rows):
    s = oracle.split_24(np.ascontiguousarray(W[rows]), "bf16")
    S = oracle.nm24_to_dense(f64(s["val"]), s["idx"])
    return oracle.apply_rows(np.arange(len(rows)), S, f64(U[rows]), f64(V), f64(X))


@pytest.mark.parametrize("m,n,r,T", [
    (300, 128, 8, 64), (128, 64, 0, 100), (257, 192, 72, 300), (64, 256, 256, 513),
    (129, 128, 16, 256), (1000, 320, 64, 70),
])
def test_prefill_small_shapes(hsl, m, n, r, T):
    L, W, U, V = build(hsl, m, n, r, m + n + r)
    X = synth.to_bf16_bits(synth.normal_f32(T, n, T))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    rows = np.arange(m)
    check_close(f64(host(Y)), ref_rows(W, U, V, X, rows), "bf16")


def test_prefill_matches_decode_path(hsl):
    """Same layer, same tokens: tensor-core path (one call of 128 tokens) and
    CUDA-core path (sixteen calls of 8) agree to bf16 output rounding."""
    L, W, U, V = build(hsl, 512, 512, 32, 7)
    X = synth.to_bf16_bits(synth.normal_f32(128, 512, 1))
    Xd = dev(X, "bf16")
    Yp = L.apply(Xd)
    Yd = torch.cat([L.apply(Xd[i:i + 8].contiguous()) for i in range(0, 128, 8)])
    a, b = f64(host(Yp)), f64(host(Yd))
    assert oracle.rel_err(a, b) <= 2 * TOL["bf16"]


def test_prefill_mlp_up_11008_2048_tokens_sampled(hsl):
    lay = MLP_UP_11008.layers[0]
    L, W, U, V = build(hsl, lay.m, lay.n, MLP_UP_11008.r, lay.seed, stand_in=True)
    X = synth.to_bf16_bits(synth.normal_f32(2048, lay.n, lay.seed + 1))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    rows = np.sort(np.random.default_rng(2).choice(lay.m, 384, replace=False))
    rows[-1] = lay.m - 1
    got = f64(host(Y))[:, rows]
    check_close(got, ref_rows(W, U, V, X, rows), "bf16")


def test_prefill_mlp_70b_4096_tokens_sampled(hsl):
    lay = MLP70B.layers[0]
    L, W, U, V = build(hsl, lay.m, lay.n, MLP70B.r, lay.seed, stand_in=True)
    X = synth.to_bf16_bits(synth.normal_f32(4096, lay.n, lay.seed + 1))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    rows = np.sort(np.random.default_rng(4).choice(lay.m, 192, replace=False))
    rows[-1] = lay.m - 1
    toks = np.sort(np.random.default_rng(5).choice(4096, 512, replace=False))
    got = f64(host(Y))[np.ix_(toks, rows)]
    check_close(got, ref_rows(W, U, V, X[toks], rows), "bf16")


def test_sparse_mma_matches_expansion_path(hsl, monkeypatch):
    """The 2:4 sparse tensor-core kernel and the kernel that expands each 2:4
    tile to dense in shared memory compute the same product."""
    L, W, U, V = build(hsl, 640, 512, 48, 13)
    X = synth.to_bf16_bits(synth.normal_f32(300, 512, 2))
    Xd = dev(X, "bf16")
    Ys = L.apply(Xd)
    monkeypatch.setenv("HSL_PREFILL_EXPAND", "1")
    Ye = L.apply(Xd)
    monkeypatch.delenv("HSL_PREFILL_EXPAND")
    L.check()
    assert oracle.rel_err(f64(host(Ys)), f64(host(Ye))) <= 2 * TOL["bf16"]
    assert oracle.rel_err(f64(host(Ys)), ref_rows(W, U, V, X, np.arange(640))) <= TOL["bf16"]


@pytest.mark.parametrize("m,n,r,T", [(1100, 256, 40, 700), (512, 128, 0, 2000), (300, 192, 256, 520)])
def test_cta_pair_kernel_parity(hsl, monkeypatch, m, n, r, T):
    """The CTA-pair sparse kernel (opt-in) against the oracle: tiles of 512 rows
    and 192 tokens with ragged rows and tokens, with and without the low-rank term."""
    L, W, U, V = build(hsl, m, n, r, m + 3 * n + r)
    X = synth.to_bf16_bits(synth.normal_f32(T, n, T + 1))
    monkeypatch.setenv("HSL_PREFILL_PAIRS", "1")
    Y = L.apply(dev(X, "bf16"))
    monkeypatch.delenv("HSL_PREFILL_PAIRS")
    L.check()
    check_close(f64(host(Y)), ref_rows(W, U, V, X, np.arange(m)), "bf16")
