"""Permutation for concentration on the GPU against the oracle: the ratio ρ
(fp64 sums, relative error ≤ 1e-12), the RCM order (identical), the permuted
copy of W (bit for bit) and the permuted apply (the layer's tolerance)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth

from gpu_util import TOL, check_close, dev, factors, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


@pytest.mark.parametrize("m,n,dtype,seed", [
    (1024, 1024, "f32", 0), (4096, 4096, "bf16", 2000), (4096, 4096, "f32", 2000),
    (5, 7, "f32", 1), (1, 9, "bf16", 2), (3, 1, "f32", 3), (1023, 1001, "f32", 4),
    (777, 333, "bf16", 5), (28672, 8192, "bf16", 5000),
])
def test_concentration_matches_oracle(hsl, m, n, dtype, seed):
    W = synth.as_storage(synth.student_t_f32(m, n, seed), dtype)
    got = hsl.concentration(dev(W, dtype))
    want = oracle.concentration(W, dtype)
    assert got == pytest.approx(want, rel=1e-12, abs=1e-15)


def test_concentration_unaligned_and_degenerate(hsl):
    W = synth.student_t_f32(64, 130, 9)
    big = dev(np.concatenate([np.zeros(1, np.float32), W.reshape(-1)]), "f32")
    assert hsl.concentration(big[1:].view(64, 130)) == pytest.approx(
        oracle.concentration(W, "f32"), rel=1e-12)
    assert hsl.concentration(torch.zeros(8, 8, device="cuda")) == 0.0
    D = np.zeros((6, 8), np.float32)
    D[:3, :4] = 1.0
    D[3:, 4:] = -2.0
    assert hsl.concentration(dev(D, "f32")) == 1.0


def _pattern(m, n, seed, p):
    mask = np.random.default_rng(seed).random((m, n)) < p
    rp = np.zeros(m + 1, np.int64)
    rp[1:] = np.cumsum(mask.sum(1))
    return rp, np.nonzero(mask)[1]


@pytest.mark.parametrize("m,n,p,seed", [(40, 30, 0.08, 1), (200, 317, 0.01, 2), (1, 5, 0.5, 3),
                                        (64, 64, 0.0, 4), (333, 129, 0.05, 5)])
def test_rcm_order_matches_oracle_on_patterns(hsl, m, n, p, seed):
    rp, col = _pattern(m, n, seed, p)
    ro, co = hsl.rcm_order(m, n, rp, col)
    wr, wc = oracle.rcm_order(m, n, rp, col)
    assert np.array_equal(ro, wr) and np.array_equal(co, wc)


@pytest.mark.parametrize("m,n,frac,seed", [(1024, 1024, 0.05, 0), (4096, 4096, 0.02, 2000)])
def test_rcm_order_of_a_split_matches_oracle(hsl, m, n, frac, seed):
    """The order of the GPU split's own S pattern (the workloads' layers)."""
    W = synth.student_t_f32(m, n, seed)
    L = hsl.Layer(m, n, 0, "csr", "f32")
    L.split(dev(W, "f32"), frac, None)
    S = L.get_sparse()
    rp, col = S["row_ptr"].cpu().numpy(), S["col"].cpu().numpy()
    ro, co = hsl.rcm_order(m, n, rp, col)
    wr, wc = oracle.rcm_order(m, n, rp, col)
    assert np.array_equal(ro, wr) and np.array_equal(co, wc)


@pytest.mark.parametrize("m,n,dtype", [(4096, 4096, "bf16"), (333, 77, "f32"), (1, 1, "bf16")])
def test_permute_bit_exact(hsl, m, n, dtype):
    W = synth.as_storage(synth.student_t_f32(m, n, m + n), dtype)
    rng = np.random.default_rng(m)
    ro, co = rng.permutation(m).astype(np.int32), rng.permutation(n).astype(np.int32)
    out = hsl.permute(dev(W, dtype), torch.from_numpy(ro).cuda(), torch.from_numpy(co).cuda())
    assert np.array_equal(host(out), oracle.permute(W, ro, co))


def test_permute_refuses_a_non_permutation(hsl):
    W = torch.zeros(4, 5, device="cuda")
    ro = torch.tensor([0, 1, 1, 3], dtype=torch.int32, device="cuda")
    co = torch.arange(5, dtype=torch.int32, device="cuda")
    with pytest.raises(hsl.HslError) as e:
        hsl.permute(W, ro, co)
    assert e.value.name == "HSL_ERR_INVALID_ARG"
    with pytest.raises(hsl.HslError):
        hsl.permute(W, torch.arange(4, dtype=torch.int32, device="cuda"),
                    torch.tensor([0, 1, 2, 3, 5], dtype=torch.int32, device="cuda"))


def test_rcm_recovers_hidden_blocks_through_the_library(hsl):
    """Two dense blocks hidden by random permutations: ρ rises to 1 once the
    library's RCM order of the pattern is applied by the library's permute."""
    rng = np.random.default_rng(7)
    B = np.zeros((512, 384), np.float32)
    B[:256, :192] = rng.standard_normal((256, 192)) * (rng.random((256, 192)) < 0.05)
    B[256:, 192:] = rng.standard_normal((256, 192)) * (rng.random((256, 192)) < 0.05)
    B[:256, 0] = 1.0
    B[0, :192] = 1.0
    B[256:, 192] = 1.0
    B[256, 192:] = 1.0
    H = B[rng.permutation(512)][:, rng.permutation(384)]
    rp, col = _pattern_of(H)
    ro, co = hsl.rcm_order(512, 384, rp, col)
    P = hsl.permute(dev(H, "f32"), torch.from_numpy(ro).cuda(), torch.from_numpy(co).cuda())
    assert hsl.concentration(dev(H, "f32")) < 0.6
    assert hsl.concentration(P) == 1.0


def _pattern_of(A):
    mask = A != 0
    rp = np.zeros(A.shape[0] + 1, np.int64)
    rp[1:] = np.cumsum(mask.sum(1))
    return rp, np.nonzero(mask)[1]


@pytest.mark.parametrize("fmt,dtype,m,n,r,T", [
    ("csr", "bf16", 1000, 768, 16, 1), ("csr", "f32", 300, 200, 8, 5),
    ("nm24", "bf16", 4096, 1024, 32, 1), ("nm24", "bf16", 4096, 1024, 32, 16),
    ("nm24", "bf16", 1100, 1024, 32, 100),
])
def test_permuted_apply_matches_oracle(hsl, fmt, dtype, m, n, r, T):
    """The layer is built from W' = W[row_order][:, col_order] (its RCM order),
    and the permuted apply returns the original order: y = P_rᵀ Ŵ' P_c x."""
    W = synth.as_storage(synth.student_t_f32(m, n, m * 3 + n), dtype)
    frac = 0.05 if fmt == "csr" else 0.5
    ref0 = oracle.split_topk(W, 0.05, dtype)
    ro, co = oracle.rcm_order(m, n, ref0["row_ptr"], ref0["col"])
    Wp = oracle.permute(W, ro, co)
    ref = oracle.split_topk(Wp, frac, dtype) if fmt == "csr" else oracle.split_24(Wp, dtype)
    R64 = oracle.bits_to_f64(ref["R"], dtype)
    U, V = factors(R64, r, dtype)
    L = hsl.Layer(m, n, r, fmt, dtype)
    Wd = hsl.permute(dev(W, dtype), torch.from_numpy(ro).cuda(), torch.from_numpy(co).cuda())
    L.split(Wd, frac, None)
    L.pack(dev(U, dtype), dev(V, dtype))
    L.set_permutation(torch.from_numpy(ro).cuda(), torch.from_numpy(co).cuda())
    X = synth.as_storage(synth.normal_f32(T, n, T), dtype)
    Y = L.apply(dev(X, dtype))
    L.check()
    f = lambda b: oracle.bits_to_f64(b, dtype)  # noqa: E731
    if fmt == "csr":
        S = oracle.csr_to_dense(m, n, ref["row_ptr"], ref["col"], f(ref["val"]))
    else:
        S = oracle.nm24_to_dense(f(ref["val"]), ref["idx"])
    Yp = oracle.apply(oracle.reconstruct(S, f(U), f(V)), f(X)[:, co])
    Yref = np.empty_like(Yp)
    Yref[:, ro] = Yp
    check_close(f(host(Y)), Yref, dtype)
    # clearing the permutation gives the permuted layer's own output
    L.set_permutation(None, None)
    check_close(f(host(L.apply(dev(X, dtype)))), oracle.apply(oracle.reconstruct(S, f(U), f(V)), f(X)),
                dtype)
