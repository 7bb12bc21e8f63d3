"""Stage 2 on the GPU (hsl_factor) against the oracle's randomized truncated
SVD given the same Gaussian test matrix Ω: singular values, the rank-r product
U Vᵀ, the residual energy ‖R − U Vᵀ‖², and U, V column by column where the
spectrum separates them; exact recovery of a planted low-rank residual; and
the whole path split → factor → pack → apply against the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth

from gpu_util import TOL, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def omega_of(n, k, seed):
    return np.random.default_rng(seed).standard_normal((n, k)).astype(np.float32)


def gpu_factor(hsl, R_bits, dtype, r, omega, q, layer_dtype="f32"):
    m, n = R_bits.shape
    L = hsl.Layer(m, n, r, "csr", layer_dtype)
    U, V, sig = L.factor(dev(R_bits, dtype), torch.from_numpy(omega).cuda(), q)
    L.check()
    torch.cuda.synchronize()
    f = lambda t: oracle.bits_to_f64(host(t), layer_dtype)  # noqa: E731
    return f(U), f(V), sig.cpu().numpy().astype(np.float64)


def oracle_factor(R64, r, omega, q):
    U, V = oracle.lowrank_randomized(R64, r, omega.astype(np.float64), power_iters=q)
    return U, V, np.einsum("ij,ij->j", U, U)   # U = U_r √Σ_r, so UᵀU = diag(σ)


def align_signs(Ug, Vg, Vo):
    s = np.sign(np.einsum("ij,ij->j", Vg, Vo))
    s[s == 0] = 1.0
    return Ug * s, Vg * s


def test_factor_planted_spectrum_matches_oracle_column_by_column(hsl):
    """A residual with distinct singular values and a gap after r: σ, U Vᵀ and
    each factor column agree with the oracle at fp32 accuracy."""
    rng = np.random.default_rng(31)
    m, n, r, k, q = 1000, 700, 12, 24, 2
    Ua, _ = np.linalg.qr(rng.standard_normal((m, n)))
    Va, _ = np.linalg.qr(rng.standard_normal((n, n)))
    s = np.concatenate([np.linspace(8, 3, r), 0.3 * np.exp(-np.arange(n - r) / 50)])
    R = ((Ua * s) @ Va.T).astype(np.float32)
    om = omega_of(n, k, 32)
    Ug, Vg, sg = gpu_factor(hsl, R, "f32", r, om, q)
    Uo, Vo, so = oracle_factor(R.astype(np.float64), r, om, q)
    assert np.allclose(sg, so, rtol=1e-5)
    Pg, Po = Ug @ Vg.T, Uo @ Vo.T
    assert np.abs(Pg - Po).max() <= 1e-5 * s[0]
    Ug, Vg = align_signs(Ug, Vg, Vo)
    assert np.abs(Ug - Uo).max() <= 1e-4 * np.abs(Uo).max()
    assert np.abs(Vg - Vo).max() <= 1e-4 * np.abs(Vo).max()


def test_factor_recovers_an_exactly_low_rank_residual(hsl):
    """R = A Bᵀ of rank 6 (integers, exact in fp32), k = 16 > rank: the
    directions beyond the rank are dropped (σ = 0, zero columns) and U Vᵀ = R."""
    rng = np.random.default_rng(33)
    m, n = 300, 200
    A = rng.integers(-3, 4, size=(m, 6)).astype(np.float32)
    B = rng.integers(-3, 4, size=(n, 6)).astype(np.float32)
    R = A @ B.T
    om = omega_of(n, 16, 34)
    Ug, Vg, sg = gpu_factor(hsl, R, "f32", 8, om, 1)
    assert np.all(sg[6:] == 0.0) and np.all(sg[:6] > 0)
    assert not Ug[:, 6:].any() and not Vg[:, 6:].any()
    assert np.abs(Ug @ Vg.T - R).max() <= 1e-5 * np.abs(R).max()
    Uo, Vo, so = oracle_factor(R.astype(np.float64), 6, om, 1)
    assert np.allclose(sg[:6], so, rtol=1e-5)


def test_factor_zero_residual(hsl):
    R = np.zeros((64, 96), np.float32)
    Ug, Vg, sg = gpu_factor(hsl, R, "f32", 4, omega_of(96, 8, 1), 1)
    assert not sg.any() and not Ug.any() and not Vg.any()


def test_factor_square1024_worked_example_residual(hsl):
    """The worked example's residual: 1024² f32 W minus its top 5 %, rank 64,
    k = 74, two power iterations (the oracle's own defaults)."""
    W = synth.student_t_f32(1024, 1024, 0)
    R = oracle.split_topk(W, 0.05, "f32")["R"].view(np.float32)   # storage bits as values
    om = omega_of(1024, 74, 35)
    Ug, Vg, sg = gpu_factor(hsl, R, "f32", 64, om, 2)
    R64 = R.astype(np.float64)
    Uo, Vo, so = oracle_factor(R64, 64, om, 2)
    assert np.allclose(sg, so, rtol=1e-5)
    # the flat tail of a noise-like spectrum makes single directions sensitive;
    # the rank-64 product and its residual energy are not
    Pg, Po = Ug @ Vg.T, Uo @ Vo.T
    assert np.abs(Pg - Po).max() <= 1e-3 * np.abs(Po).max()
    eg = np.linalg.norm(R64 - Pg) ** 2
    eo = np.linalg.norm(R64 - Po) ** 2
    assert abs(eg - eo) <= 1e-5 * eo


def test_factor_bf16_up_projection_residual(hsl):
    """11008×4096 bf16 layer: the 2:4 residual, rank 64, k = 74, one power
    iteration; factors stored as bf16 (rounded once from fp32)."""
    m, n, r, k = 11008, 4096, 64, 74
    W = synth.to_bf16_bits(synth.student_t_f32(m, n, 3000))
    R = oracle.split_24(W, "bf16")["R"]
    om = omega_of(n, k, 36)
    Ug, Vg, sg = gpu_factor(hsl, R, "bf16", r, om, 1, layer_dtype="bf16")
    R64 = oracle.bits_to_f64(R, "bf16")
    Uo, Vo, so = oracle_factor(R64, r, om, 1)
    assert np.allclose(sg, so, rtol=1e-5)
    rows = np.random.default_rng(37).choice(m, 256, replace=False)
    Pg, Po = Ug[rows] @ Vg.T, Uo[rows] @ Vo.T
    # bf16 storage of U and V: 2^-8 relative per factor entry
    assert np.abs(Pg - Po).max() <= 2e-2 * np.abs(Po).max()
    assert np.linalg.norm(Pg - Po) <= 1e-2 * np.linalg.norm(Po)


def test_split_factor_pack_apply_against_the_oracle(hsl):
    """The whole compression on the GPU (split, factor, pack) and the apply,
    against the oracle's split, randomized SVD (same Ω) and dense product."""
    m, n, r, k = 2048, 1024, 32, 42
    W = synth.to_bf16_bits(synth.student_t_f32(m, n, 41))
    L = hsl.Layer(m, n, r, "csr", "bf16")
    Rd = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    L.split(dev(W, "bf16"), 0.05, Rd)
    om = omega_of(n, k, 42)
    U, V, _ = L.factor(Rd, torch.from_numpy(om).cuda(), 2)
    L.pack(U, V)
    X = synth.to_bf16_bits(synth.normal_f32(4, n, 43))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    ref = oracle.split_topk(W, 0.05, "bf16")
    f = lambda b: oracle.bits_to_f64(b, "bf16")  # noqa: E731
    Uo, Vo = oracle.lowrank_randomized(f(ref["R"]), r, om.astype(np.float64), power_iters=2)
    Uo, Vo = f(synth.to_bf16_bits(Uo.astype(np.float32))), f(synth.to_bf16_bits(Vo.astype(np.float32)))
    S = oracle.csr_to_dense(m, n, ref["row_ptr"], ref["col"], f(ref["val"]))
    Yref = oracle.apply(oracle.reconstruct(S, Uo, Vo), f(X))
    assert oracle.rel_err(f(host(Y)), Yref) <= TOL["bf16"]


def test_factor_argument_checks(hsl):
    L = hsl.Layer(64, 32, 8, "csr", "f32")
    R = torch.zeros(64, 32, device="cuda")
    with pytest.raises(hsl.HslError) as e:
        L.factor(R, torch.zeros(32, 4, device="cuda"))          # k < r
    assert e.value.name == "HSL_ERR_UNSUPPORTED"
    with pytest.raises(hsl.HslError) as e:
        L.factor(R, torch.zeros(32, 40, device="cuda"))         # k > min(m, n)
    assert e.value.name == "HSL_ERR_UNSUPPORTED"
    with pytest.raises(ValueError):
        L.factor(R, torch.zeros(31, 8, device="cuda"))
