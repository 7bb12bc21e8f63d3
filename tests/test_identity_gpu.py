"""Identity probe: applying a layer to X = I_n (n tokens, token t the unit
vector e_t) makes the GPU write Y[t] = Ŵ e_t, the t-th column of Ŵ, so Y = Ŵᵀ,
compared element by element with the oracle's reconstruction Ŵ = S + U Vᵀ.

With one unit vector per token, S·e_t is a single stored value and z = Vᵀ e_t
is a row of V (exact in bf16, so the tensor-core path's hi/lo pair is exact
too); the only rounding is the fp32 sum of U·z and the output's conversion to
the layer dtype.  Bound per element: half an output ulp of |Ŵ_ij| (2⁻⁸·|Ŵ_ij|
for bf16, 2⁻²⁴·|Ŵ_ij| for f32) plus the fp32 sum's error, taken as one fp32 ulp
per addition, r·2⁻²³·Σ_c|U_ic V_jc| (a tensor-core adder may truncate rather
than round).  A wrong index or a dropped group costs a whole |S_ij| and fails."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth

from gpu_util import csr_dense_rows, dev, factors, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def identity(n, dtype):
    return synth.as_storage(np.eye(n, dtype=np.float32), dtype)


def check(Y, S64, U, V, dtype):
    f = lambda b: oracle.bits_to_f64(b, dtype)  # noqa: E731
    U64, V64 = f(U), f(V)
    W_hat = oracle.reconstruct(S64, U64, V64)
    got = f(host(Y)).T                             # Y = Ŵᵀ
    ulp = 2.0 ** -7 if dtype == "bf16" else 2.0 ** -23   # spacing at 1.0 (8 / 24 significant bits)
    bound = 0.5 * ulp * np.abs(W_hat) + U64.shape[1] * 2.0 ** -23 * (np.abs(U64) @ np.abs(V64).T) + 1e-30
    bad = np.argwhere(np.abs(got - W_hat) > bound)
    assert bad.size == 0, f"{len(bad)} entries of Ŵ off, first at {tuple(bad[0])}"


@pytest.mark.parametrize("m,n,r", [(1024, 1024, 64), (700, 512, 32)])
def test_identity_reconstructs_w_hat_2to4_tensor_cores(hsl, m, n, r):
    """bf16 2:4, n ≥ 65 tokens: the sparse-MMA prefill kernel."""
    W = synth.to_bf16_bits(synth.student_t_f32(m, n, m + n))
    ref = oracle.split_24(W, "bf16")
    U, V = factors(oracle.bits_to_f64(ref["R"], "bf16"), r, "bf16")
    L = hsl.Layer(m, n, r, "nm24", "bf16")
    L.split(dev(W, "bf16"), 0.5, None)
    L.pack(dev(U, "bf16"), dev(V, "bf16"))
    Y = L.apply(dev(identity(n, "bf16"), "bf16"))
    L.check()
    S = oracle.nm24_to_dense(oracle.bits_to_f64(ref["val"], "bf16"), ref["idx"])
    check(Y, S, U, V, "bf16")


def test_identity_reconstructs_w_hat_csr_tensor_cores(hsl):
    """bf16 CSR at 5 %, 1024 tokens: the kernel that decompresses S into
    shared memory for the dense MMA."""
    m = n = 1024
    W = synth.to_bf16_bits(synth.student_t_f32(m, n, 7))
    ref = oracle.split_topk(W, 0.05, "bf16")
    U, V = factors(oracle.bits_to_f64(ref["R"], "bf16"), 64, "bf16")
    L = hsl.Layer(m, n, 64, "csr", "bf16")
    L.split(dev(W, "bf16"), 0.05, None)
    L.pack(dev(U, "bf16"), dev(V, "bf16"))
    Y = L.apply(dev(identity(n, "bf16"), "bf16"))
    L.check()
    S = csr_dense_rows(ref["row_ptr"], ref["col"], oracle.bits_to_f64(ref["val"], "bf16"),
                       np.arange(m), n)
    check(Y, S, U, V, "bf16")


def test_identity_reconstructs_w_hat_square1024_f32(hsl):
    """The worked example's layer (1024², 5 %, r = 64, f32): the CUDA-core
    decode kernel, 16 tokens per pass."""
    m = n = 1024
    W = synth.student_t_f32(m, n, 0)
    ref = oracle.split_topk(W, 0.05, "f32")
    U, V = factors(oracle.bits_to_f64(ref["R"], "f32"), 64, "f32", exact=True)
    L = hsl.Layer(m, n, 64, "csr", "f32")
    L.split(dev(W, "f32"), 0.05, None)
    L.pack(dev(U, "f32"), dev(V, "f32"))
    Y = L.apply(dev(identity(n, "f32"), "f32"))
    L.check()
    S = csr_dense_rows(ref["row_ptr"], ref["col"], oracle.bits_to_f64(ref["val"], "f32"), np.arange(m), n)
    check(Y, S, U, V, "f32")
