"""Pins for the CPU oracle, against things other than the oracle itself.

* the pages' worked example (tests/golden/worked_example.json);
* O(N²) brute-force ranking on tiny inputs with ties, ±0, ±Inf, denormals;
* a planted sparse + exactly-rank-r matrix that must be recovered exactly;
* Eckart–Young with the singular values taken from a different routine;
* textbook CSR SpMV (scipy) for r = 0, a pure-Python triple loop for the apply;
* mutation checks: a plausible bug planted in a copy of the oracle, on the CPU,
  must fail these pins.
"""
import json
import math
import os
import struct

import numpy as np
import pytest
import scipy.sparse
import torch

import oracle
from sparse_rank_linear_03_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

def _f32_of_bits(u32):
    return struct.unpack("<f", struct.pack("<I", int(u32)))[0]


def _py_value(bits, dtype):
    """Independent scalar decode (struct), not the oracle's bit helpers."""
    if dtype == "f32":
        return _f32_of_bits(int(bits))
    return _f32_of_bits(int(bits) << 16)


def brute_selected(flat_bits, dtype, k):
    """Set of linear indices ranked < k by (|w| desc, index asc), O(N²)."""
    mags = [abs(_py_value(b, dtype)) for b in flat_bits]
    sel = set()
    for e, me in enumerate(mags):
        ahead = 0
        for f, mf in enumerate(mags):
            if mf > me or (mf == me and f < e):
                ahead += 1
        if ahead < k:
            sel.add(e)
    return sel


def tie_heavy_f32(m, n, seed):
    rng = np.random.default_rng(seed)
    v = rng.integers(-3, 4, size=(m, n)).astype(np.float32)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, 1e-40, -1e-40, 1e-45, 3.0, -3.0],
                        dtype=np.float32)
    pos = rng.choice(m * n, size=min(len(specials), m * n), replace=False)
    v.reshape(-1)[pos] = specials[: len(pos)]
    return v


def tie_heavy_bf16(m, n, seed):
    rng = np.random.default_rng(seed)
    # small alphabet of bf16 bit patterns incl. ±0, ±Inf, a denormal, and ties
    alphabet = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x8001,
                         0x3F80, 0xBF80, 0x4000, 0xC000, 0x3F80, 0x3C00], dtype=np.uint16)
    return alphabet[rng.integers(0, len(alphabet), size=(m, n))]


# ---------------------------------------------------------------- worked example

def test_worked_example_counts():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    pc = oracle.param_counts(g["m"], g["n"], g["frac"], g["r"])
    assert pc["dense"] == g["dense"]
    assert pc["sparse"] == g["sparse"]
    assert g["factor_each"][0] * g["factor_each"][1] * 2 == g["factor"] == pc["factor"]
    assert pc["total"] == g["total"]
    assert f"{pc['reduction']:.1f}x" == g["reduction_as_printed"]
    assert round(100 * pc["residual_footprint_reduction"]) == g["residual_footprint_reduction_as_printed_pct"]
    assert pc["residual"] == 996_148


def test_worked_example_split_size():
    """The oracle's split of the 1024² seed-0 layer keeps exactly 52,428."""
    W = synth.student_t_f32(1024, 1024, 0)
    s = oracle.split_topk(W, 0.05, "f32")
    assert s["k"] == 52_428 == len(s["col"]) == s["row_ptr"][-1]


@pytest.mark.parametrize("frac,m,n,k", [
    (0.02, 4096, 4096, 335_544),       # attention workload, stated count
    (0.03, 4096, 4096, 503_316),
    (0.03, 11008, 4096, 1_352_663),
    (0.05, 28672, 8192, 11_744_051),
    (0.0, 5, 5, 0), (-1.0, 5, 5, 0), (1.0, 5, 5, 25), (2.0, 5, 5, 25),
])
def test_topk_count_floor(frac, m, n, k):
    assert oracle.topk_count(frac, m, n) == k


def test_nm24_counts():
    assert oracle.nm24_count(11008, 4096) == 22_544_384
    assert oracle.nm24_count(28672, 8192) == 117_440_512


# ---------------------------------------------------------------- split by brute force

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("seed", [1, 2])
def test_split_topk_bruteforce_8x8(dtype, seed):
    W = tie_heavy_f32(8, 8, seed) if dtype == "f32" else tie_heavy_bf16(8, 8, seed)
    bits = W.view(np.uint32) if dtype == "f32" else W
    flat = bits.reshape(-1)
    for k in range(0, 65):
        frac = k / 64.0
        s = oracle.split_topk(W, frac, dtype)
        assert s["k"] == k
        sel = brute_selected(flat, dtype, k)
        rows = np.repeat(np.arange(8), np.diff(s["row_ptr"]))
        got = set((rows * 8 + s["col"]).tolist())
        assert got == sel, k
        # canonical CSR: columns strictly ascending in each row
        for i in range(8):
            c = s["col"][s["row_ptr"][i]:s["row_ptr"][i + 1]]
            assert np.all(np.diff(c) > 0)
        # values are the original bits; residual is W with +0.0 at kept positions
        lin = rows * 8 + s["col"]
        assert np.array_equal(s["val"], flat[lin])
        R = s["R"].reshape(-1)
        for e in range(64):
            assert R[e] == (0 if e in sel else flat[e])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 9), (9, 1), (3, 7), (5, 4), (2, 2)])
def test_split_topk_bruteforce_shapes(shape, dtype):
    """Single rows and columns, rows left empty, every k: the CSR rows come from
    the brute-force selection (empty rows have equal row_ptr entries)."""
    m, n = shape
    W = tie_heavy_f32(m, n, 11 + m) if dtype == "f32" else tie_heavy_bf16(m, n, 11 + m)
    flat = (W.view(np.uint32) if dtype == "f32" else W).reshape(-1)
    for k in range(0, m * n + 1):
        s = oracle.split_topk(W, k / (m * n), dtype)
        assert s["k"] == k
        sel = brute_selected(flat, dtype, k)
        per_row = [sum(1 for e in sel if e // n == i) for i in range(m)]
        assert np.array_equal(np.diff(s["row_ptr"]), per_row)
        rows = np.repeat(np.arange(m), np.diff(s["row_ptr"]))
        assert set((rows * n + s["col"]).tolist()) == sel


def test_split_topk_nan_rejected():
    W = np.ones((3, 3), dtype=np.float32)
    W[1, 1] = np.nan
    with pytest.raises(ValueError):
        oracle.split_topk(W, 0.5, "f32")


def test_split_24_bruteforce_all_groups():
    vals = np.array([0.0, -0.0, 1.0, -1.0, 2.0, np.inf, 1e-40], dtype=np.float32)
    groups = np.array(np.meshgrid(*([np.arange(len(vals))] * 4), indexing="ij")).reshape(4, -1).T
    W = vals[groups]                       # [2401, 4]
    W = np.concatenate([W, W[::-1]], axis=1)  # n = 8: two groups per row
    s = oracle.split_24(W, "f32")
    bits = W.view(np.uint32)
    for i in range(W.shape[0]):
        for g in range(2):
            grp = bits[i, 4 * g:4 * g + 4]
            mags = [abs(_py_value(b, "f32")) for b in grp]
            keep = [e for e in range(4)
                    if sum(1 for f in range(4) if mags[f] > mags[e] or (mags[f] == mags[e] and f < e)) < 2]
            nib = int(s["idx"][i, g])
            assert [nib & 3, nib >> 2] == keep
            assert list(s["val"][i, 2 * g:2 * g + 2]) == [grp[keep[0]], grp[keep[1]]]
            for e in range(4):
                assert s["R"][i, 4 * g + e] == (0 if e in keep else grp[e])


def test_split_24_bf16_matches_f32_reading():
    """bf16 and f32 inputs with the same values give the same selection."""
    W = synth.student_t_f32(16, 64, 11)
    Wb = synth.to_bf16_bits(W)
    Wf = oracle.bits_to_f64(Wb, "bf16").astype(np.float32)
    a = oracle.split_24(Wb, "bf16")
    b = oracle.split_24(Wf, "f32")
    assert np.array_equal(a["idx"], b["idx"])


def test_split_invariants_student_t():
    W = synth.student_t_f32(64, 96, 5)
    s = oracle.split_topk(W, 0.07, "f32")
    k = s["k"]
    rp = s["row_ptr"]
    assert rp[0] == 0 and rp[-1] == k and np.all(np.diff(rp) >= 0)
    rows = np.repeat(np.arange(64), np.diff(rp))
    lin = rows * 96 + s["col"]
    mask = np.zeros(64 * 96, bool)
    mask[lin] = True
    mag = np.abs(W.astype(np.float64)).reshape(-1)
    assert mag[mask].min() >= mag[~mask].max()
    t = mag[mask].min()
    sel_t = np.nonzero(mask & (mag == t))[0]
    uns_t = np.nonzero(~mask & (mag == t))[0]
    if len(uns_t):
        assert sel_t.max() < uns_t.min()
    # S ⊕ R reproduces W bit for bit
    R = s["R"].reshape(-1).view(np.uint32)
    Wb = W.reshape(-1).view(np.uint32)
    assert np.array_equal(np.where(mask, Wb, R), Wb)
    assert np.all(R[mask] == 0)
    dense = oracle.csr_to_dense(64, 96, rp, s["col"], oracle.bits_to_f64(s["val"], "f32"))
    assert np.array_equal(dense + oracle.bits_to_f64(s["R"], "f32"), W.astype(np.float64))


def test_split_24_invariants():
    W = synth.to_bf16_bits(synth.student_t_f32(32, 128, 9))
    s = oracle.split_24(W, "bf16")
    i0, i1 = s["idx"] & 3, s["idx"] >> 2
    assert np.all(i0 < i1)
    D = oracle.nm24_to_dense(oracle.bits_to_f64(s["val"], "bf16"), s["idx"])
    assert np.all((D != 0).reshape(32, 32, 4).sum(-1) <= 2)
    assert np.array_equal(D + oracle.bits_to_f64(s["R"], "bf16"), oracle.bits_to_f64(W, "bf16"))


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_special_cases():
    cases = {
        0x3F800000: 0x3F80,   # 1.0
        0x3F808000: 0x3F80,   # halfway, even stays
        0x3F818000: 0x3F82,   # halfway, odd rounds up
        0x3F808001: 0x3F81,   # just above halfway
        0x7F7FFFFF: 0x7F80,   # max float rounds to +Inf
        0xFF800000: 0xFF80,   # -Inf
        0x80000000: 0x8000,   # -0
        0x00000001: 0x0000,   # tiny denormal rounds to +0
        0x00018000: 0x0002,   # denormal halfway, odd → up
    }
    u = np.array(list(cases.keys()), dtype=np.uint32)
    got = oracle.f32_to_bf16_bits(u.view(np.float32))
    assert [int(x) for x in got] == list(cases.values())
    nan = oracle.f32_to_bf16_bits(np.array([np.nan], dtype=np.float32))[0]
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F) != 0


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(3).standard_normal(100_000).astype(np.float32) * 1e3
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16_bits(x), ref)


# ---------------------------------------------------------------- low rank

def _planted(m, n, r, seed):
    """W = S0 + A Bᵀ exactly representable in float32, A zero on rows I."""
    rng = np.random.default_rng(seed)
    A = rng.integers(-2, 3, size=(m, r)).astype(np.float64)
    B = rng.integers(-2, 3, size=(n, r)).astype(np.float64)
    I = rng.choice(m, size=m // 4, replace=False)
    A[I] = 0.0
    L = A @ B.T
    S0 = np.zeros((m, n))
    for i in I:
        cols = rng.choice(n, size=3, replace=False)
        S0[i, cols] = rng.choice([-1, 1], size=3) * (1000.0 + rng.integers(0, 50, size=3))
    W = (S0 + L).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), S0 + L)
    return W, S0, L


def test_exact_reconstruction_planted():
    m, n, r = 48, 40, 3
    W, S0, L = _planted(m, n, r, 21)
    k = int(np.count_nonzero(S0))
    s = oracle.split_topk(W, k / (m * n) + 1e-12, "f32")
    assert s["k"] == k
    D = oracle.csr_to_dense(m, n, s["row_ptr"], s["col"], oracle.bits_to_f64(s["val"], "f32"))
    assert np.array_equal(D, S0)
    R = oracle.bits_to_f64(s["R"], "f32")
    assert np.array_equal(R, L)
    U, V = oracle.lowrank_svd(R, r)
    W_hat = oracle.reconstruct(D, U, V)
    assert np.abs(W_hat - W).max() <= 1e-12 * np.abs(W).max()
    X = np.random.default_rng(1).standard_normal((5, n))
    assert oracle.rel_err(oracle.apply(W_hat, X), X @ W.astype(np.float64).T) < 1e-12


def test_eckart_young_with_eigvalsh():
    R = np.random.default_rng(7).standard_normal((40, 30))
    r = 6
    U, V = oracle.lowrank_svd(R, r)
    lam = np.sort(np.linalg.eigvalsh(R.T @ R))[::-1]      # σ² from a different routine
    err = np.linalg.norm(R - U @ V.T, "fro") ** 2
    assert abs(err - lam[r:].sum()) <= 1e-10 * lam.sum()
    # √σ split: UᵀU = VᵀV = diag(σ)
    sig = np.sqrt(lam[:r])
    assert np.allclose(U.T @ U, np.diag(sig), atol=1e-10)
    assert np.allclose(V.T @ V, np.diag(sig), atol=1e-10)


def test_lowrank_rank_above_min_dimension_is_exact_and_zero_padded():
    R = np.random.default_rng(17).standard_normal((5, 12))
    U, V = oracle.lowrank_svd(R, 9)
    assert U.shape == (5, 9) and V.shape == (12, 9)
    assert not U[:, 5:].any() and not V[:, 5:].any()
    assert np.abs(U @ V.T - R).max() < 1e-12


def test_randomized_matches_exact_on_low_rank():
    rng = np.random.default_rng(8)
    R = rng.standard_normal((60, 5)) @ rng.standard_normal((5, 50))
    omega = rng.standard_normal((50, 5 + 8))
    U, V = oracle.lowrank_randomized(R, 5, omega)
    assert np.abs(U @ V.T - R).max() < 1e-10 * np.abs(R).max()


def test_randomized_matches_exact_truncation_across_a_gap():
    """Spectrum with a clear gap after r: with power iterations the randomized
    factors reproduce the exact truncated SVD (Eckart–Young optimum), and keep
    the √σ balance UᵀU = VᵀV = diag(σ)."""
    rng = np.random.default_rng(21)
    m, n, r = 120, 90, 7
    Ua, _ = np.linalg.qr(rng.standard_normal((m, n)))
    Va, _ = np.linalg.qr(rng.standard_normal((n, n)))
    sig = np.concatenate([np.linspace(10, 5, r), np.linspace(1, 0.01, n - r)])
    R = (Ua * sig) @ Va.T
    omega = rng.standard_normal((n, r + 6))
    # subspace error decays like (σ_{r+1}/σ_r)^(2q+1) = 0.2^13 ≈ 1e-9 at q = 6
    U, V = oracle.lowrank_randomized(R, r, omega, power_iters=6)
    Ue, Ve = oracle.lowrank_svd(R, r)
    assert np.abs(U @ V.T - Ue @ Ve.T).max() < 1e-7 * sig[0]
    assert np.allclose(np.diag(U.T @ U), sig[:r], rtol=1e-9)
    assert np.allclose(U.T @ U, V.T @ V, atol=1e-9)
    err = np.linalg.norm(R - U @ V.T, "fro") ** 2
    assert abs(err - (sig[r:] ** 2).sum()) <= 1e-9 * (sig ** 2).sum()


def test_randomized_without_power_iterations_is_worse_but_bounded():
    """q = 0 on a flat tail: a valid rank-r factorisation whose residual is no
    better than the optimum (Eckart–Young) and within the HMT bound's order."""
    rng = np.random.default_rng(22)
    R = rng.standard_normal((80, 60))
    r = 5
    omega = rng.standard_normal((60, r + 10))
    U, V = oracle.lowrank_randomized(R, r, omega, power_iters=0)
    s = np.linalg.svd(R, compute_uv=False)
    err = np.linalg.norm(R - U @ V.T, "fro") ** 2
    assert err >= (s[r:] ** 2).sum() * (1 - 1e-12)
    assert err <= 2.0 * (s[r:] ** 2).sum()


# ---------------------------------------------------------------- apply

def _triple_loop(S, U, V, X):
    m, n = len(S), len(S[0])
    r = len(U[0]) if m and U else 0
    Y = []
    for x in X:
        z = [sum(V[j][c] * x[j] for j in range(n)) for c in range(r)]
        Y.append([sum(S[i][j] * x[j] for j in range(n)) + sum(U[i][c] * z[c] for c in range(r))
                  for i in range(m)])
    return np.array(Y)


@pytest.mark.parametrize("r", [0, 1, 3])
@pytest.mark.parametrize("shape", [(8, 8), (7, 9), (9, 5)])
def test_apply_triple_loop(r, shape):
    m, n = shape
    rng = np.random.default_rng(100 + r)
    W = rng.standard_normal((m, n)).astype(np.float32)
    s = oracle.split_topk(W, 0.3, "f32")
    D = oracle.csr_to_dense(m, n, s["row_ptr"], s["col"], oracle.bits_to_f64(s["val"], "f32"))
    U = rng.standard_normal((m, r))
    V = rng.standard_normal((n, r))
    X = rng.standard_normal((3, n))
    Y = oracle.apply(oracle.reconstruct(D, U, V), X)
    assert Y.shape == (3, m)
    ref = _triple_loop(D.tolist(), U.tolist(), V.tolist(), X.tolist())
    assert np.abs(Y - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_apply_r0_is_textbook_spmv():
    W = synth.student_t_f32(50, 70, 3)
    s = oracle.split_topk(W, 0.1, "f32")
    vals = oracle.bits_to_f64(s["val"], "f32")
    A = scipy.sparse.csr_matrix((vals, s["col"], s["row_ptr"]), shape=(50, 70))
    X = np.random.default_rng(4).standard_normal((4, 70))
    D = oracle.csr_to_dense(50, 70, s["row_ptr"], s["col"], vals)
    Y = oracle.apply(oracle.reconstruct(D, np.zeros((50, 0)), np.zeros((70, 0))), X)
    assert np.abs(Y - (A @ X.T).T).max() < 1e-13


def test_apply_k0_is_two_dense_products():
    rng = np.random.default_rng(5)
    U, V, X = rng.standard_normal((30, 4)), rng.standard_normal((20, 4)), rng.standard_normal((6, 20))
    Y = oracle.apply(oracle.reconstruct(np.zeros((30, 20)), U, V), X)
    assert np.abs(Y - (X @ V) @ U.T).max() < 1e-12


def test_apply_frac1_is_dense():
    W = synth.student_t_f32(12, 10, 6)
    s = oracle.split_topk(W, 1.0, "f32")
    assert s["k"] == 120 and not s["R"].view(np.uint32).any()
    D = oracle.csr_to_dense(12, 10, s["row_ptr"], s["col"], oracle.bits_to_f64(s["val"], "f32"))
    X = np.random.default_rng(2).standard_normal((2, 10))
    assert np.array_equal(D, W.astype(np.float64))
    assert np.abs(oracle.apply(D, X) - X @ W.astype(np.float64).T).max() < 1e-14


def test_apply_24_matches_dense_definition():
    W = synth.to_bf16_bits(synth.student_t_f32(10, 16, 12))
    s = oracle.split_24(W, "bf16")
    D = oracle.nm24_to_dense(oracle.bits_to_f64(s["val"], "bf16"), s["idx"])
    Wf = oracle.bits_to_f64(W, "bf16")
    X = np.random.default_rng(0).standard_normal((2, 16))
    ref = [[sum(D[i][j] * x[j] for j in range(16)) for i in range(10)] for x in X]
    assert np.abs(oracle.apply(D, X) - np.array(ref)).max() < 1e-14
    # kept entries are the two largest of each group
    for i in range(10):
        for g in range(4):
            grp = np.abs(Wf[i, 4 * g:4 * g + 4])
            kept = np.abs(D[i, 4 * g:4 * g + 4])[D[i, 4 * g:4 * g + 4] != 0]
            assert sorted(kept)[-1] <= grp.max()


def test_apply_rows_matches_full():
    rng = np.random.default_rng(9)
    D = rng.standard_normal((20, 15))
    U, V = rng.standard_normal((20, 3)), rng.standard_normal((15, 3))
    X = rng.standard_normal((4, 15))
    rows = np.array([0, 5, 19])
    full = oracle.apply(oracle.reconstruct(D, U, V), X)
    assert np.abs(oracle.apply_rows(rows, D[rows], U, V, X) - full[:, rows]).max() < 1e-13


def test_rel_err_definition():
    Y = np.array([[1.0, 2.0], [0.0, 0.0]])
    R = np.array([[1.0, 4.0], [0.0, 0.0]])
    assert oracle.rel_err(Y, R) == 0.5
    assert oracle.rel_err(np.zeros((0, 3)), np.zeros((0, 3))) == 0.0


def test_elem_rel_err_definition():
    """Hand-computed: row max 10, floor 1e-3 → denominators max(|y*|, 0.01)."""
    R = np.array([[10.0, -0.001, 2.0, 0.0]])
    Y = np.array([[10.1, 0.0, 2.0, 0.002]])
    # 0.1/10, 0.001/0.01, 0/2, 0.002/0.01 → 0.2 from the last column
    assert oracle.elem_rel_err(Y, R) == pytest.approx(0.2, rel=1e-12)
    assert oracle.elem_rel_err(Y[:, :3], R[:, :3]) == pytest.approx(0.1, rel=1e-12)
    # a zero reference row is compared absolutely; empty input is 0
    assert oracle.elem_rel_err(np.array([[0.5, 0.0]]), np.zeros((1, 2))) == 0.5
    assert oracle.elem_rel_err(np.zeros((0, 3)), np.zeros((0, 3))) == 0.0
    # never below the normwise measure (each denominator is at most the row max)
    rng = np.random.default_rng(3)
    A = rng.standard_normal((4, 50))
    B = A + 1e-3 * rng.standard_normal((4, 50))
    assert oracle.elem_rel_err(B, A) >= oracle.rel_err(B, A)


# ---------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_tie_break_bug(monkeypatch):
    """Ties to the HIGHER index (a plausible bug) must fail the brute force."""
    real = oracle.hss.np.lexsort

    def wrong(keys):
        lin, negmag = keys
        return real((-lin, negmag))

    W = tie_heavy_f32(8, 8, 1)
    monkeypatch.setattr(oracle.hss.np, "lexsort", wrong)
    s = oracle.split_topk(W, 20 / 64, "f32")
    monkeypatch.undo()
    rows = np.repeat(np.arange(8), np.diff(s["row_ptr"]))
    got = set((rows * 8 + s["col"]).tolist())
    assert got != brute_selected(W.view(np.uint32).reshape(-1), "f32", 20)


def test_pins_catch_planted_transpose_bug():
    """Y = X Ŵ (transposed operand) must fail the triple-loop pin."""
    rng = np.random.default_rng(1)
    D = rng.standard_normal((7, 9))
    U, V = rng.standard_normal((7, 2)), rng.standard_normal((9, 2))
    X = rng.standard_normal((2, 9))
    ref = _triple_loop(D.tolist(), U.tolist(), V.tolist(), X.tolist())
    W_hat = oracle.reconstruct(D, U, V)
    with pytest.raises(ValueError):
        _ = X @ W_hat             # shapes refuse the transposed product
    sq = rng.standard_normal((6, 6))
    Xs = rng.standard_normal((2, 6))
    assert not np.allclose(Xs @ sq, oracle.apply(sq, Xs))


def test_pins_catch_dropped_lowrank_term():
    rng = np.random.default_rng(2)
    D = rng.standard_normal((8, 8))
    U, V = rng.standard_normal((8, 1)), rng.standard_normal((8, 1))
    X = rng.standard_normal((1, 8))
    ref = _triple_loop(D.tolist(), U.tolist(), V.tolist(), X.tolist())
    assert np.abs(oracle.apply(D, X) - ref).max() > 1e-6       # S-only is wrong
    assert np.abs(oracle.apply(oracle.reconstruct(D, U, V), X) - ref).max() < 1e-12


# ---------------------------------------------------------------- concentration and RCM

def test_concentration_hand_example():
    """4×4, quadrants split at row 2 and column 2: diagonal blocks hold
    |1|+|-2|+|3|+|4| + |5|+|6|+|-7|+|8| = 36 of a total 36 + 10 = 46."""
    W = np.array([[1, -2, 1, 0],
                  [3, 4, 0, -2],
                  [0, 3, 5, 6],
                  [-4, 0, -7, 8]], dtype=np.float32)
    assert oracle.concentration(W, "f32") == pytest.approx(36 / 46, rel=1e-15)


@pytest.mark.parametrize("m,n", [(4, 4), (5, 7), (1, 9), (512, 512), (3, 1)])
def test_concentration_uniform_magnitude_closed_form(m, n):
    """Equal |w| everywhere: ρ is the share of entries in the two blocks,
    (⌊m/2⌋⌊n/2⌋ + ⌈m/2⌉⌈n/2⌉)/(m n), whatever the signs."""
    rng = np.random.default_rng(m * n)
    W = np.where(rng.random((m, n)) < 0.5, -0.25, 0.25).astype(np.float32)
    mh, nh = m // 2, n // 2
    want = (mh * nh + (m - mh) * (n - nh)) / (m * n)
    assert oracle.concentration(W, "f32") == pytest.approx(want, rel=1e-15)
    assert oracle.concentration(synth.to_bf16_bits(W), "bf16") == pytest.approx(want, rel=1e-15)


def test_concentration_block_extremes_and_zero():
    D = np.zeros((6, 8), np.float32)
    D[:3, :4] = 1.0
    D[3:, 4:] = -2.0
    assert oracle.concentration(D, "f32") == 1.0
    assert oracle.concentration(D[:, ::-1].copy(), "f32") == 0.0     # mass off the diagonal
    assert oracle.concentration(np.zeros((3, 3), np.float32), "f32") == 0.0


def test_permute_definition():
    W = np.arange(12, dtype=np.float32).reshape(3, 4)
    ro, co = [2, 0, 1], [3, 1, 0, 2]
    P = oracle.permute(W, ro, co)
    for k in range(3):
        for l in range(4):
            assert P[k, l] == W[ro[k], co[l]]


def _csr_of(mask):
    m = mask.shape[0]
    rp = np.zeros(m + 1, np.int64)
    rp[1:] = np.cumsum(mask.sum(axis=1))
    return rp, np.nonzero(mask)[1]


def test_rcm_returns_permutations():
    rng = np.random.default_rng(5)
    mask = rng.random((40, 30)) < 0.08
    ro, co = oracle.rcm_order(40, 30, *_csr_of(mask))
    assert sorted(ro.tolist()) == list(range(40)) and sorted(co.tolist()) == list(range(30))


def _scipy_rcm_bipartite(mask):
    from scipy.sparse import bmat, csr_matrix
    from scipy.sparse.csgraph import reverse_cuthill_mckee
    S = csr_matrix(mask.astype(np.int8))
    G = bmat([[None, S], [S.T, None]], format="csr")
    G.sort_indices()
    return reverse_cuthill_mckee(G, symmetric_mode=True)


def test_rcm_matches_scipy_where_the_start_is_unique():
    """scipy's reverse_cuthill_mckee on the bipartite graph follows the same
    steps; its choice among equal-degree start vertices is its sort's, so the
    comparison uses connected graphs whose smallest degree is held by one
    vertex (neighbour ties are broken by vertex number on both sides)."""
    rng = np.random.default_rng(11)
    checked = 0
    for trial in range(400):
        m, n = int(rng.integers(3, 25)), int(rng.integers(3, 25))
        mask = rng.random((m, n)) < rng.uniform(0.1, 0.5)
        deg = np.concatenate([mask.sum(1), mask.sum(0)])
        if deg.min() == 0 or (deg == deg.min()).sum() != 1:
            continue
        from scipy.sparse import csr_matrix, bmat
        from scipy.sparse.csgraph import connected_components
        G = bmat([[None, csr_matrix(mask)], [csr_matrix(mask).T, None]])
        if connected_components(G, directed=False)[0] != 1:
            continue
        ref = _scipy_rcm_bipartite(mask)
        ro, co = oracle.rcm_order(m, n, *_csr_of(mask))
        assert np.array_equal(ro, ref[ref < m]), trial
        assert np.array_equal(co, ref[ref >= m] - m), trial
        checked += 1
    assert checked >= 20


def test_rcm_gathers_a_hidden_block_diagonal():
    """Two dense blocks hidden by random row and column permutations: the
    RCM order makes each block contiguous again, so ρ of the permuted
    pattern is 1 (the blocks are the two diagonal quadrants)."""
    rng = np.random.default_rng(2)
    B = np.zeros((16, 12), bool)
    B[:8, :6] = rng.random((8, 6)) < 0.6
    B[8:, 6:] = rng.random((8, 6)) < 0.6
    B[0, :6] = B[8, 6:] = True          # every row and column has an entry
    B[:8, 0] = B[8:, 6] = True
    pr, pc = rng.permutation(16), rng.permutation(12)
    H = B[pr][:, pc]
    ro, co = oracle.rcm_order(16, 12, *_csr_of(H))
    P = oracle.permute(H.astype(np.float32), ro, co)
    assert oracle.concentration(P, "f32") == 1.0
    assert oracle.concentration(H.astype(np.float32), "f32") < 0.8


def test_pins_catch_an_unreversed_order():
    """Cuthill–McKee without the final reversal (a plausible slip) fails the
    scipy comparison on a graph whose order is not a palindrome."""
    rng = np.random.default_rng(4)
    for _ in range(500):
        mask = rng.random((9, 7)) < 0.35
        deg = np.concatenate([mask.sum(1), mask.sum(0)])
        if deg.min() > 0 and (deg == deg.min()).sum() == 1:
            break
    ref = _scipy_rcm_bipartite(mask)
    ro, co = oracle.rcm_order(9, 7, *_csr_of(mask))
    assert np.array_equal(ro, ref[ref < 9])
    assert not np.array_equal(ro[::-1], ref[ref < 9])
