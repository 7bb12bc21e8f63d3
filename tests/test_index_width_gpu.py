"""Column-index widths of the packed CSR S (hsl_set_index_bits): 8-bit deltas
with a 16-bit base per vector, 16-bit and 32-bit columns give the same apply,
checked against the float64 oracle (the layer's tolerances) and bit for bit on
integer inputs; filler entries for gaps over 255 columns; 32-bit columns for
n ≥ 65535; refusals where a width cannot hold the pattern."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth

from gpu_util import check_close, csr_dense_rows, dev, factors, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def layer(hsl, m, n, r, frac, dtype, bits, seed):
    W = synth.as_storage(synth.student_t_f32(m, n, seed), dtype)
    ref = oracle.split_topk(W, frac, dtype)
    U, V = factors(oracle.bits_to_f64(ref["R"], dtype), r, dtype, seed)
    L = hsl.Layer(m, n, r, "csr", dtype)
    L.set_index_bits(bits)
    L.split(dev(W, dtype), frac, None)
    L.pack(dev(U, dtype), dev(V, dtype))
    return L, ref, U, V


def check(hsl, L, ref, U, V, dtype, T, seed):
    m, n = L.m, L.n
    X = synth.as_storage(synth.normal_f32(T, n, seed), dtype)
    Y = L.apply(dev(X, dtype))
    L.check()
    f = lambda b: oracle.bits_to_f64(b, dtype)  # noqa: E731
    S = csr_dense_rows(ref["row_ptr"], ref["col"], f(ref["val"]), np.arange(m), n)
    check_close(f(host(Y)), oracle.apply_rows(np.arange(m), S, f(U), f(V), f(X)), dtype)


@pytest.mark.parametrize("bits", [8, 16, 32])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("m,n,frac,r", [(1000, 768, 0.03, 16), (129, 77, 0.2, 3), (64, 4096, 0.002, 8)])
def test_widths_match_oracle(hsl, bits, dtype, m, n, frac, r):
    """The last shape has gaps far beyond 255 columns: the 8-bit layout fills them."""
    L, ref, U, V = layer(hsl, m, n, r, frac, dtype, bits, m + n + bits)
    for T in (1, 3, 16):
        check(hsl, L, ref, U, V, dtype, T, T)


def test_8bit_fillers_on_far_apart_columns(hsl):
    """Rows whose entries sit at columns 0, 300, 1000, 4095 (gaps of 300,
    700 and 3095 need 1, 2 and 12 fillers), imported as given."""
    m, n = 40, 4096
    cols = np.tile(np.array([0, 300, 1000, 4095], np.int32), m)
    rp = np.arange(0, 4 * m + 1, 4, dtype=np.int32)
    vals = synth.to_bf16_bits(np.random.default_rng(1).standard_normal(4 * m).astype(np.float32))
    L = hsl.Layer(m, n, 0, "csr", "bf16")
    L.set_index_bits(8)
    L.set_sparse_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(cols).cuda(), dev(vals, "bf16"))
    L.pack(None, None)
    X = synth.to_bf16_bits(synth.normal_f32(2, n, 3))
    Y = L.apply(dev(X, "bf16"))
    L.check()
    f = lambda b: oracle.bits_to_f64(b, "bf16")  # noqa: E731
    S = oracle.csr_to_dense(m, n, rp, cols, f(vals))
    check_close(f(host(Y)), oracle.apply(S, f(X)), "bf16")


def test_8bit_refuses_descending_columns(hsl):
    L = hsl.Layer(4, 64, 0, "csr", "bf16")
    L.set_index_bits(8)
    rp = torch.tensor([0, 2, 2, 2, 2], dtype=torch.int32, device="cuda")
    col = torch.tensor([9, 3], dtype=torch.int32, device="cuda")
    L.set_sparse_csr(rp, col, torch.ones(2, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(hsl.HslError) as e:
        L.pack(None, None)
    assert e.value.name == "HSL_ERR_UNSUPPORTED"
    L.set_index_bits(16)            # the same S packs with 16-bit columns
    L.pack(None, None)


def test_32bit_columns_for_wide_rows(hsl):
    """n = 70000 ≥ 65535: 32-bit columns are the default; 16- and 8-bit refused."""
    m, n = 48, 70000
    with pytest.raises(hsl.HslError):
        hsl.Layer(m, n, 4, "csr", "bf16").set_index_bits(16)
    L, ref, U, V = layer(hsl, m, n, 4, 0.01, "bf16", 0, 5)
    check(hsl, L, ref, U, V, "bf16", 1, 6)


def test_8bit_group_of_a_7b_layer(hsl):
    """One 7B layer's seven projections with 8-bit columns, applied as a group."""
    shapes = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    built = [layer(hsl, m, n, 16, 0.03, "bf16", 8, 700 + i) for i, (m, n) in enumerate(shapes)]
    g = hsl.Group([b[0] for b in built])
    Xs = [synth.to_bf16_bits(synth.normal_f32(1, n, 710 + i)) for i, (m, n) in enumerate(shapes)]
    Ys = [torch.empty(1, m, dtype=torch.bfloat16, device="cuda") for m, n in shapes]
    g.apply([dev(x, "bf16") for x in Xs], Ys)
    torch.cuda.synchronize()
    f = lambda b: oracle.bits_to_f64(b, "bf16")  # noqa: E731
    for (m, n), (L, ref, U, V), X, Y in zip(shapes, built, Xs, Ys):
        rows = np.sort(np.random.default_rng(m + n).choice(m, 400, replace=False))
        S = csr_dense_rows(ref["row_ptr"], ref["col"], f(ref["val"]), rows, n)
        check_close(f(host(Y))[:, rows], oracle.apply_rows(rows, S, f(U), f(V), f(X)), "bf16")
    g.close()


def test_group_refuses_mixed_widths(hsl):
    a = layer(hsl, 64, 64, 2, 0.1, "bf16", 8, 1)[0]
    b = layer(hsl, 64, 64, 2, 0.1, "bf16", 16, 2)[0]
    with pytest.raises(hsl.HslError) as e:
        hsl.Group([a, b])
    assert e.value.name == "HSL_ERR_UNSUPPORTED"
