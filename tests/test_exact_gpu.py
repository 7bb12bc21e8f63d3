"""Exact-arithmetic parity of the apply kernels with the float64 oracle.

Every input is a small integer or half-integer, chosen so that every product
and every partial sum the kernels form in fp32 is exact in any order of
summation (all magnitudes stay far below 2^24), and z = Vᵀx is an integer
below 2^16, so that the tensor-core path's bf16 hi/lo split of z is exact as
well.  The kernel's fp32 result then equals the oracle's float64 y* exactly,
and its one rounding, to the bf16 output (round to nearest even), is the
oracle's rounding of y*: the outputs must agree bit for bit, element by
element, with zero error.  A single mis-decoded 2:4 group, a swapped metadata
nibble, a dropped chunk or a lost U·z term changes some y* by at least 0.5,
which the comparison sees wherever the bf16 output can hold the difference
(|y*| < 128 for most outputs here; elsewhere both sides round the same way).

Shapes are the workloads' own (the 70B MLP layer 28672×8192 with r = 256, the
11008×4096 up-projection with r = 64, the 4096² attention projection with
r = 128, one 7B layer's seven projections as a group) in the launch
configurations the library picks for them; outputs are compared on sampled
rows (all of a row's tokens), which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth

from gpu_util import csr_dense_rows, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def ints(shape, seed, values, probs, dtype):
    """Storage bits of an array whose entries are drawn from `values`."""
    rng = np.random.default_rng(seed)
    v = np.asarray(values, dtype=np.float32)[rng.choice(len(values), size=shape, p=probs)]
    return synth.as_storage(v, dtype)


def weights(m, n, seed, dtype, csr):
    """Signed magnitudes {0.5, 1, 2} (2:4), or with a rare 4 on top (top-k)."""
    if csr:
        mags, p = [0.5, 1.0, 2.0, 4.0], [0.6, 0.3, 0.08, 0.02]
    else:
        mags, p = [0.5, 1.0, 2.0], [0.4, 0.4, 0.2]
    vals = [s * v for v in mags for s in (1.0, -1.0)]
    probs = [q / 2 for q in p for _ in (0, 1)]
    return ints((m, n), seed, vals, probs, dtype)


def tokens(t, n, seed, dtype):
    return ints((t, n), seed, [-1.0, 0.0, 1.0], [0.25, 0.5, 0.25], dtype)


def factors(m, n, r, seed, dtype):
    """V dense in {-1, 0, 1}; U with about four nonzeros per row."""
    V = ints((n, r), seed, [-1.0, 0.0, 1.0], [0.25, 0.5, 0.25], dtype)
    pu = min(0.5, 4.0 / max(r, 1))
    U = ints((m, r), seed + 1, [-1.0, 0.0, 1.0], [pu / 2, 1 - pu, pu / 2], dtype)
    return U, V


def expected_bits(S_rows64, U, V, X, rows, dtype):
    """Exact y* on the sampled rows, rounded once to the layer dtype."""
    f = lambda b: oracle.bits_to_f64(b, dtype)  # noqa: E731
    Y = oracle.apply_rows(np.arange(len(rows)), S_rows64, f(U[rows]), f(V), f(X))
    assert np.all(np.abs(Y) < 2 ** 24) and np.array_equal(Y, np.round(2 * Y) / 2)
    Y32 = Y.astype(np.float32)
    return oracle.f32_to_bf16_bits(Y32) if dtype == "bf16" else Y32.view(np.uint32)


def got_bits(Y, rows, dtype):
    h = host(Y)[:, rows]
    return h if dtype == "bf16" else h.view(np.uint32)


def assert_exact(got, want):
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} outputs differ, first at (token, row) {tuple(bad[0])}"


def sample_rows(m, count, seed):
    rows = np.sort(np.random.default_rng(seed).choice(m, size=min(count, m), replace=False))
    rows[0], rows[-1] = 0, m - 1
    return np.unique(rows)


def build_24(hsl, m, n, r, seed, dtype="bf16"):
    W = weights(m, n, seed, dtype, csr=False)
    U, V = factors(m, n, r, seed + 10, dtype)
    L = hsl.Layer(m, n, r, "nm24", dtype)
    L.split(dev(W, dtype), 0.5, None)
    L.pack(dev(U, dtype), dev(V, dtype))
    return L, W, U, V


def rows_24(W, rows, dtype):
    s = oracle.split_24(np.ascontiguousarray(W[rows]), dtype)
    return oracle.nm24_to_dense(oracle.bits_to_f64(s["val"], dtype), s["idx"])


def check_24(hsl, L, W, U, V, T, seed, rows, dtype="bf16", tok=None):
    X = tokens(T, W.shape[1], seed, dtype)
    Y = L.apply(dev(X, dtype))
    L.check()
    torch.cuda.synchronize()
    Xs = X if tok is None else X[tok]
    want = expected_bits(rows_24(W, rows, dtype), U, V, Xs, rows, dtype)
    got = got_bits(Y, rows, dtype)
    assert_exact(got if tok is None else got[tok], want)


# ---------------------------------------------------------------- 2:4


def test_exact_2to4_70b_batch1(hsl):
    """28672×8192, r = 256, batch 1: the single-launch bulk-copy decode kernel."""
    m, n, r = 28672, 8192, 256
    L, W, U, V = build_24(hsl, m, n, r, 501)
    check_24(hsl, L, W, U, V, 1, 502, sample_rows(m, 3000, 503))


def test_exact_2to4_70b_prefill_4096(hsl):
    """Same layer, 4096 tokens: the tcgen05 sparse-MMA prefill kernel."""
    m, n, r = 28672, 8192, 256
    L, W, U, V = build_24(hsl, m, n, r, 511)
    tok = np.sort(np.random.default_rng(512).choice(4096, 384, replace=False))
    check_24(hsl, L, W, U, V, 4096, 513, sample_rows(m, 384, 514), tok=tok)


@pytest.mark.parametrize("T", [1, 4, 16, 2048])
def test_exact_2to4_11008(hsl, T):
    """11008×4096, r = 64 at every batch of the workload (bulk-copy decode,
    register-fed decode, the batch-16 path and the 2048-token prefill)."""
    m, n, r = 11008, 4096, 64
    L, W, U, V = build_24(hsl, m, n, r, 521)
    tok = None if T <= 16 else np.sort(np.random.default_rng(T).choice(T, 256, replace=False))
    check_24(hsl, L, W, U, V, T, 522 + T, sample_rows(m, 1500 if T <= 16 else 256, 523), tok=tok)


@pytest.mark.parametrize("T", [2, 8, 33, 64, 700])
def test_exact_2to4_ragged_rows(hsl, T):
    """1100 rows (a partial last row tile) × 1024: the split-K kernel at 2-64
    tokens (units of two K-blocks dealt over all SMs) and the default prefill
    kernel at 700 tokens, every output compared bit for bit."""
    m, n, r = 1100, 1024, 40
    L, W, U, V = build_24(hsl, m, n, r, 535)
    check_24(hsl, L, W, U, V, T, 536 + T, np.arange(m))


@pytest.mark.parametrize("env", ["HSL_PREFILL_EXPAND", "HSL_PREFILL_PAIRS"])
def test_exact_2to4_alternate_prefill_kernels(hsl, monkeypatch, env):
    """The expansion kernel and the CTA-pair kernel, exact on a ragged shape."""
    m, n, r = 1100, 1024, 40
    L, W, U, V = build_24(hsl, m, n, r, 531)
    monkeypatch.setenv(env, "1")
    check_24(hsl, L, W, U, V, 700, 532, np.arange(m))
    monkeypatch.delenv(env)


def test_exact_2to4_f32_layer(hsl):
    """An f32 2:4 layer: fp32 output, compared bit for bit."""
    m, n, r = 700, 1024, 16
    L, W, U, V = build_24(hsl, m, n, r, 541, dtype="f32")
    for T in (1, 5, 40):
        check_24(hsl, L, W, U, V, T, 542 + T, np.arange(m), dtype="f32")


# ---------------------------------------------------------------- CSR


def build_csr(hsl, m, n, r, frac, seed, dtype="bf16"):
    W = weights(m, n, seed, dtype, csr=True)
    U, V = factors(m, n, r, seed + 10, dtype)
    L = hsl.Layer(m, n, r, "csr", dtype)
    L.split(dev(W, dtype), frac, None)
    L.pack(dev(U, dtype), dev(V, dtype))
    ref = oracle.split_topk(W, frac, dtype)
    return L, ref, U, V


def csr_rows(ref, rows, n, dtype):
    return csr_dense_rows(ref["row_ptr"], ref["col"], oracle.bits_to_f64(ref["val"], dtype), rows, n)


@pytest.mark.parametrize("T", [1, 4, 16, 2048])
def test_exact_csr_attn4096(hsl, T):
    """4096², 2 % top-k, r = 128 at batch 1/4/16 (the CSR decode kernel) and
    2048 tokens (the tensor-core path that decompresses S block by block)."""
    m = n = 4096
    L, ref, U, V = build_csr(hsl, m, n, 128, 0.02, 551)
    X = tokens(T, n, 552 + T, "bf16")
    Y = L.apply(dev(X, "bf16"))
    L.check()
    rows = sample_rows(m, 2000 if T <= 16 else 256, 553)
    tok = np.arange(T) if T <= 16 else np.sort(np.random.default_rng(T).choice(T, 256, replace=False))
    assert_exact(got_bits(Y, rows, "bf16")[tok],
                 expected_bits(csr_rows(ref, rows, n, "bf16"), U, V, X[tok], rows, "bf16"))


def test_exact_csr_7b_layer_group(hsl):
    """One 7B layer's seven projections (3 % top-k, r = 128) as one group."""
    shapes = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    built = [build_csr(hsl, m, n, 128, 0.03, 560 + i) for i, (m, n) in enumerate(shapes)]
    g = hsl.Group([b[0] for b in built])
    Xs = [tokens(1, n, 570 + i, "bf16") for i, (m, n) in enumerate(shapes)]
    Ys = [torch.empty(1, m, dtype=torch.bfloat16, device="cuda") for m, n in shapes]
    for _ in range(2):
        g.apply([dev(x, "bf16") for x in Xs], Ys)
        torch.cuda.synchronize()
        for (m, n), (L, ref, U, V), X, Y in zip(shapes, built, Xs, Ys):
            rows = sample_rows(m, 600, m + n)
            assert_exact(got_bits(Y, rows, "bf16"),
                         expected_bits(csr_rows(ref, rows, n, "bf16"), U, V, X, rows, "bf16"))
    g.close()


@pytest.mark.parametrize("T", [1, 3])
def test_exact_csr_square1024_f32(hsl, T):
    """The 1024² f32 layer at 5 %, r = 64: fp32 output, bit for bit."""
    m = n = 1024
    L, ref, U, V = build_csr(hsl, m, n, 64, 0.05, 581, dtype="f32")
    X = tokens(T, n, 582, "f32")
    Y = L.apply(dev(X, "f32"))
    L.check()
    rows = np.arange(m)
    assert_exact(got_bits(Y, rows, "f32"),
                 expected_bits(csr_rows(ref, rows, n, "f32"), U, V, X, rows, "f32"))


@pytest.mark.parametrize("bits", [8, 32])
def test_exact_csr_other_column_widths(hsl, bits):
    """The 4096² layer with 8-bit delta or 32-bit columns, batch 1 and 4."""
    m = n = 4096
    W = weights(m, n, 591, "bf16", csr=True)
    U, V = factors(m, n, 128, 601, "bf16")
    L = hsl.Layer(m, n, 128, "csr", "bf16")
    L.set_index_bits(bits)
    L.split(dev(W, "bf16"), 0.02, None)
    L.pack(dev(U, "bf16"), dev(V, "bf16"))
    ref = oracle.split_topk(W, 0.02, "bf16")
    rows = sample_rows(m, 2000, 592)
    for T in (1, 4):
        X = tokens(T, n, 593 + T, "bf16")
        Y = L.apply(dev(X, "bf16"))
        L.check()
        assert_exact(got_bits(Y, rows, "bf16"),
                     expected_bits(csr_rows(ref, rows, n, "bf16"), U, V, X, rows, "bf16"))
