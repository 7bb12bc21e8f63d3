"""Parity of the GPU apply y = S x + U (Vᵀ x) with the float64 oracle.

Tolerance (max over tokens of the normwise relative error): 1e-5 for f32
layers, 1e-2 for bf16 layers (fp32 accumulation, bf16 output).  The
element-wise error (denominator max(|y*|, 1e-3·max|y*|)) is checked beside it:
1e-3 for f32, 1e-2 for bf16."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth
from sparse_rank_linear_03_b200.configs import ATTN4096, MLP70B, MLP_UP_11008, PR1, STACK7B

from gpu_util import ELEM_TOL, TOL, csr_dense_rows, dev, factors, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def f64(bits, dtype):
    return oracle.bits_to_f64(bits, dtype)


class Case:
    """A layer built through the oracle (S, U, V) and the same layer on the GPU."""

    def __init__(self, hsl, m, n, r, fmt, dtype, frac, seed, split_dtype=None, gpu_split=True,
                 exact_svd=False, skew=False):
        split_dtype = split_dtype or dtype
        Wf = synth.student_t_f32(m, n, seed)
        if skew:
            Wf = synth.skew_columns(Wf, seed)
        W = synth.as_storage(Wf, split_dtype)
        self.m, self.n, self.r, self.fmt, self.dtype = m, n, r, fmt, dtype
        if fmt == "csr":
            ref = oracle.split_topk(W, frac, split_dtype)
            vals = ref["val"]
            if split_dtype != dtype:
                vals = (oracle.f32_to_bf16_bits(vals.view(np.float32)) if dtype == "bf16"
                        else f64(vals, "bf16").astype(np.float32))
            self.rp, self.col, self.val = ref["row_ptr"], ref["col"], vals
        else:
            ref = oracle.split_24(W, split_dtype)
            vals = ref["val"]
            if split_dtype != dtype:
                vals = (oracle.f32_to_bf16_bits(vals.view(np.float32)) if dtype == "bf16"
                        else f64(vals, "bf16").astype(np.float32))
            self.nmv, self.nmi = vals, ref["idx"]
        R64 = f64(ref["R"], split_dtype)
        self.U, self.V = factors(R64, r, dtype, seed, exact=exact_svd)
        self.L = hsl.Layer(m, n, r, fmt, dtype)
        if gpu_split:
            self.L.split(dev(W, split_dtype), frac if fmt == "csr" else 0.5, None)
        elif fmt == "csr":
            self.L.set_sparse_csr(torch.from_numpy(self.rp).cuda(), torch.from_numpy(self.col).cuda(),
                                  dev(self.val, dtype))
        else:
            self.L.set_sparse_nm24(dev(self.nmv, dtype), torch.from_numpy(self.nmi).cuda())
        self.L.pack(dev(self.U, dtype), dev(self.V, dtype))
        self.L.check()

    def s_rows(self, rows):
        if self.fmt == "csr":
            return csr_dense_rows(self.rp, self.col, f64(self.val, self.dtype), rows, self.n)
        return oracle.nm24_to_dense(f64(self.nmv[rows], self.dtype), self.nmi[rows])

    def ref(self, Xbits, rows=None):
        rows = np.arange(self.m) if rows is None else rows
        return oracle.apply_rows(rows, self.s_rows(rows), f64(self.U, self.dtype),
                                 f64(self.V, self.dtype), f64(Xbits, self.dtype))

    def x(self, batch, seed):
        return synth.as_storage(synth.normal_f32(batch, self.n, seed), self.dtype)


def err_of(case, Y, Xb, rows=None):
    """Normwise error against the oracle (returned, compared by the caller);
    the element-wise error is checked against its own bound here."""
    Yh = f64(host(Y), case.dtype)
    if rows is not None:
        Yh = Yh[:, rows]
    ref = case.ref(Xb, rows)
    el = oracle.elem_rel_err(Yh, ref)
    assert el <= ELEM_TOL[case.dtype], f"element-wise error {el:.3e}"
    return oracle.rel_err(Yh, ref)


# ---------------------------------------------------------------- the workloads

def test_square1024_f32_csr_batch1(hsl):
    lay = PR1.layers[0]
    c = Case(hsl, lay.m, lay.n, PR1.r, "csr", "f32", PR1.frac, lay.seed, exact_svd=True)
    Xb = c.x(1, lay.seed + 1)
    Y = c.L.apply(dev(Xb, "f32"))
    assert err_of(c, Y, Xb) <= TOL["f32"]


@pytest.mark.parametrize("batch", ATTN4096.batches)
def test_attn4096_bf16_csr(hsl, batch):
    lay = ATTN4096.layers[0]
    c = Case(hsl, lay.m, lay.n, ATTN4096.r, "csr", "bf16", ATTN4096.frac, lay.seed,
             split_dtype="f32")
    Xb = c.x(batch, lay.seed + 1)
    Y = c.L.apply(dev(Xb, "bf16"))
    assert err_of(c, Y, Xb) <= TOL["bf16"]


@pytest.mark.parametrize("batch", [1, 4, 16])
def test_mlp_up_11008_bf16_nm24(hsl, batch):
    lay = MLP_UP_11008.layers[0]
    c = Case(hsl, lay.m, lay.n, MLP_UP_11008.r, "nm24", "bf16", 0.5, lay.seed)
    Xb = c.x(batch, lay.seed + 1)
    Y = c.L.apply(dev(Xb, "bf16"))
    assert err_of(c, Y, Xb) <= TOL["bf16"]


def test_mlp_70b_bf16_nm24_batch1_sampled_rows(hsl):
    lay = MLP70B.layers[0]
    m, n, r = lay.m, lay.n, MLP70B.r
    W = synth.to_bf16_bits(synth.student_t_f32(m, n, lay.seed))
    L = hsl.Layer(m, n, r, "nm24", "bf16")
    L.split(dev(W, "bf16"), 0.5, None)
    Uf, Vf = synth.stand_in_factors(m, n, r, lay.seed + 2)
    U, V = synth.to_bf16_bits(Uf), synth.to_bf16_bits(Vf)
    L.pack(dev(U, "bf16"), dev(V, "bf16"))
    Xb = synth.to_bf16_bits(synth.normal_f32(1, n, lay.seed + 1))
    Y = L.apply(dev(Xb, "bf16"))
    rows = np.sort(np.random.default_rng(3).choice(m, size=256, replace=False))
    rows[-1] = m - 1
    ref = oracle.split_24(np.ascontiguousarray(W[rows]), "bf16")
    S = oracle.nm24_to_dense(f64(ref["val"], "bf16"), ref["idx"])
    Yref = oracle.apply_rows(np.arange(len(rows)), S, f64(U[rows], "bf16"), f64(V, "bf16"),
                             f64(Xb, "bf16"))
    assert oracle.rel_err(f64(host(Y), "bf16")[:, rows], Yref) <= TOL["bf16"]


def test_llama7b_stack_group_two_layers(hsl):
    """The 7-projection layer shape, two layers, applied as one group."""
    cases = [Case(hsl, l.m, l.n, STACK7B.r, "csr", "bf16", STACK7B.frac, l.seed, split_dtype="f32")
             for l in STACK7B.layers[:14]]
    g = hsl.Group([c.L for c in cases])
    Xs = [c.x(1, 100 + i) for i, c in enumerate(cases)]
    Xd = [dev(x, "bf16") for x in Xs]
    Yd = [torch.empty(1, c.m, dtype=torch.bfloat16, device="cuda") for c in cases]
    for rep in range(2):
        g.apply(Xd, Yd)
        torch.cuda.synchronize()
        for c, x, y in zip(cases, Xs, Yd):
            assert err_of(c, y, x) <= TOL["bf16"]
    g.close()


# ---------------------------------------------------------------- shapes and edges

@pytest.mark.parametrize("fmt", ["csr", "nm24"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape,r", [((37, 52), 0), ((200, 100), 1), ((129, 260), 8),
                                     ((513, 1000), 3), ((1, 64), 5), ((1000, 16), 24)])
@pytest.mark.parametrize("batch", [1, 3, 17])
def test_small_shapes(hsl, fmt, dtype, shape, r, batch):
    m, n = shape
    c = Case(hsl, m, n, r, fmt, dtype, 0.07, m * 31 + n)
    Xb = c.x(batch, 5)
    Y = c.L.apply(dev(Xb, dtype))
    assert err_of(c, Y, Xb) <= TOL[dtype]


@pytest.mark.parametrize("fmt", ["csr", "nm24"])
def test_imported_sparse_matches_split(hsl, fmt):
    c = Case(hsl, 300, 512, 16, fmt, "bf16", 0.05, 9, gpu_split=False)
    Xb = c.x(4, 2)
    assert err_of(c, c.L.apply(dev(Xb, "bf16")), Xb) <= TOL["bf16"]


def test_empty_rows_and_k0(hsl):
    """k = 0 (only the low-rank term) and rows of S with no entries."""
    c = Case(hsl, 64, 96, 4, "csr", "f32", 0.0, 1)
    Xb = c.x(2, 3)
    assert err_of(c, c.L.apply(dev(Xb, "f32")), Xb) <= TOL["f32"]
    c2 = Case(hsl, 64, 96, 0, "csr", "f32", 0.002, 2)    # most rows empty, r = 0
    assert err_of(c2, c2.L.apply(dev(Xb, "f32")), Xb) <= TOL["f32"]


def test_skewed_columns(hsl):
    c = Case(hsl, 512, 1024, 32, "csr", "bf16", 0.03, 4, skew=True)
    Xb = c.x(1, 8)
    assert err_of(c, c.L.apply(dev(Xb, "bf16")), Xb) <= TOL["bf16"]


def test_host_pointers(hsl):
    """X and Y in host memory (pageable and pinned) are staged by the library."""
    c = Case(hsl, 256, 512, 8, "csr", "f32", 0.05, 6)
    Xb = c.x(3, 4)
    ref = c.ref(Xb)
    Xh = torch.from_numpy(Xb.copy())
    Yh = torch.empty(3, 256, dtype=torch.float32)
    c.L.apply(Xh, Yh)
    assert oracle.rel_err(Yh.numpy().astype(np.float64), ref) <= TOL["f32"]
    Xp = Xh.pin_memory()
    Yp = torch.empty(3, 256, dtype=torch.float32).pin_memory()
    c.L.apply(Xp, Yp)
    torch.cuda.synchronize()
    assert oracle.rel_err(Yp.numpy().astype(np.float64), ref) <= TOL["f32"]


def test_not_ready_after_resplit(hsl):
    c = Case(hsl, 32, 64, 2, "csr", "f32", 0.1, 3)
    W = dev(synth.student_t_f32(32, 64, 3), "f32")
    c.L.split(W, 0.1, None)
    with pytest.raises(hsl.HslError) as e:
        c.L.apply(dev(c.x(1, 0), "f32"))
    assert e.value.name == "HSL_ERR_NOT_READY"


def test_bad_imported_column_reported(hsl):
    L = hsl.Layer(4, 8, 0, "csr", "f32")
    rp = torch.tensor([0, 1, 1, 1, 2], dtype=torch.int32, device="cuda")
    col = torch.tensor([3, 8], dtype=torch.int32, device="cuda")      # 8 is out of range
    val = torch.tensor([1.0, 2.0], dtype=torch.float32, device="cuda")
    L.set_sparse_csr(rp, col, val)
    L.pack(None, None)
    with pytest.raises(hsl.HslError) as e:
        L.check()
    assert e.value.name == "HSL_ERR_INVALID_ARG"


# ---------------------------------------------------------------- batch-1 CSR, both kernels

@pytest.fixture(params=["regs", "bulk"])
def csr_kernel(request, monkeypatch):
    """The register-fed (default) and the bulk-copy fed batch-1 CSR kernels."""
    if request.param == "bulk":
        monkeypatch.setenv("HSL_DECODE_CSR", "bulk")
    else:
        monkeypatch.delenv("HSL_DECODE_CSR", raising=False)
    return request.param


def _import_csr(hsl, m, n, rp, col, vals, dtype="bf16", r=0, seed=0):
    L = hsl.Layer(m, n, r, "csr", dtype)
    L.set_sparse_csr(torch.from_numpy(np.asarray(rp, np.int32)).cuda(),
                     torch.from_numpy(np.asarray(col, np.int32)).cuda(), dev(vals, dtype))
    rng = np.random.default_rng(seed)
    U = synth.as_storage((0.05 * rng.standard_normal((m, r))).astype(np.float32), dtype)
    V = synth.as_storage((0.05 * rng.standard_normal((n, r))).astype(np.float32), dtype)
    L.pack(dev(U, dtype), dev(V, dtype))
    return L, U, V


def test_csr_batch1_long_rows_and_empty_rows(hsl, csr_kernel):
    """Rows longer than a streamed chunk (read from global memory), rows with
    no entries, and ordinary rows between them."""
    m, n = 300, 8192
    rng = np.random.default_rng(12)
    lens = rng.integers(0, 60, size=m)
    lens[::7] = 0
    lens[5], lens[150], lens[299] = 5000, 8192, 4033
    rp = np.zeros(m + 1, np.int64)
    rp[1:] = np.cumsum(lens)
    col = np.concatenate([np.sort(rng.choice(n, size=l, replace=False)) for l in lens]).astype(np.int32)
    vals = synth.to_bf16_bits(rng.standard_normal(int(rp[-1])).astype(np.float32))
    L, U, V = _import_csr(hsl, m, n, rp, col, vals, r=8, seed=3)
    X = synth.to_bf16_bits(synth.normal_f32(1, n, 4))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    Sd = oracle.csr_to_dense(m, n, rp, col, f64(vals, "bf16"))
    ref = oracle.apply(oracle.reconstruct(Sd, f64(U, "bf16"), f64(V, "bf16")), f64(X, "bf16"))
    assert oracle.rel_err(f64(host(Y), "bf16"), ref) <= TOL["bf16"]
    assert oracle.elem_rel_err(f64(host(Y), "bf16"), ref) <= ELEM_TOL["bf16"]


def test_csr_batch1_many_rows_per_cta(hsl, csr_kernel):
    """1.3 M rows of 16 columns: each CTA's range is longer than the window of
    row starts it stages, so it runs in several sub-parts."""
    m, n = 1_300_000, 16
    c = Case(hsl, m, n, 4, "csr", "f32", 0.1, 13)
    Xb = c.x(1, 14)
    rows = np.sort(np.random.default_rng(15).choice(m, 4000, replace=False))
    rows[-1] = m - 1
    assert err_of(c, c.L.apply(dev(Xb, "f32")), Xb, rows) <= TOL["f32"]


@pytest.mark.parametrize("bits", [8, 16, 32])
def test_csr_batch1_bulk_and_register_kernels_agree(hsl, monkeypatch, bits):
    """The bulk-copy fed and the register-fed batch-1 CSR kernels sum each row
    in different orders; they agree to bf16 output rounding."""
    c = Case(hsl, 3000, 2048, 16, "csr", "bf16", 0.03, 16)
    c.L.set_index_bits(bits)
    c.L.pack(dev(c.U, "bf16"), dev(c.V, "bf16"))
    X = dev(c.x(1, 17), "bf16")
    monkeypatch.setenv("HSL_DECODE_CSR", "bulk")
    a = f64(host(c.L.apply(X)), "bf16")
    monkeypatch.delenv("HSL_DECODE_CSR")
    b = f64(host(c.L.apply(X)), "bf16")
    assert oracle.rel_err(a, b) <= 2 ** -7


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_csr_batch17_last_token_alone(hsl, csr_kernel, dtype):
    """17 tokens: a pass of 16, then the 17th alone through the batch-1 kernel,
    which must read and write that token's rows (offset 16), not the first."""
    c = Case(hsl, 513, 1000, 3, "csr", dtype, 0.07, 513 * 31 + 1000)
    Xb = c.x(17, 5)
    assert err_of(c, c.L.apply(dev(Xb, dtype)), Xb) <= TOL[dtype]
