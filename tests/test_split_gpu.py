"""Bit-exact parity of the GPU split (top-k CSR and 2:4) with the oracle."""
import numpy as np
import pytest
import torch

import oracle
from sparse_rank_linear_03_b200 import synth
from sparse_rank_linear_03_b200.configs import ATTN4096, MLP70B, MLP_UP_11008, PR1

from gpu_util import as_bits, check_csr_equal, dev, host, ref_values

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsl():
    from sparse_rank_linear_03_b200 import hsl as mod
    return mod


def tie_heavy(m, n, seed, dtype):
    rng = np.random.default_rng(seed)
    if dtype == "bf16":
        alphabet = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x8001, 0x3F80, 0xBF80,
                             0x4000, 0xC000, 0x3C00, 0x3C01], dtype=np.uint16)
        return alphabet[rng.integers(0, len(alphabet), size=(m, n))]
    v = rng.integers(-3, 4, size=(m, n)).astype(np.float32)
    sp = np.array([0.0, -0.0, np.inf, -np.inf, 1e-40, -1e-40, 1e-45], np.float32)
    v.reshape(-1)[rng.choice(m * n, size=min(m * n, 64), replace=False)] = \
        sp[rng.integers(0, len(sp), size=min(m * n, 64))]
    return v


def run_topk(hsl, W_bits, w_dtype, layer_dtype, frac, with_residual=True):
    m, n = W_bits.shape
    L = hsl.Layer(m, n, 0, "csr", layer_dtype)
    Wd = dev(W_bits, w_dtype)
    R = torch.empty_like(Wd) if with_residual else None
    L.split(Wd, frac, R)
    L.check()
    got = L.get_sparse()
    torch.cuda.synchronize()
    return L, got, R


def assert_topk_parity(hsl, W_bits, w_dtype, layer_dtype, frac):
    L, got, R = run_topk(hsl, W_bits, w_dtype, layer_dtype, frac)
    ref = oracle.split_topk(W_bits, frac, w_dtype)
    assert L.nnz() == ref["k"]
    refv = dict(ref)
    refv["val"] = ref_values(ref["val"], w_dtype, layer_dtype)
    check_csr_equal(got, refv, layer_dtype)
    assert np.array_equal(as_bits(host(R)).reshape(-1), as_bits(ref["R"]).reshape(-1)), \
        "residual differs"
    L.close()


# ---------------------------------------------------------------- top-k, the workloads

def test_topk_square1024_f32_five_percent(hsl):
    """The 1024² worked-example layer: 52,428 kept, bit-exact."""
    lay = PR1.layers[0]
    W = synth.student_t_f32(lay.m, lay.n, lay.seed)
    assert_topk_parity(hsl, W, "f32", "f32", PR1.frac)


def test_topk_attn4096_f32_master_to_bf16_values(hsl):
    """4096² at 2 %: split on the fp32 master, values stored as bf16 (335,544 kept)."""
    lay = ATTN4096.layers[0]
    W = synth.student_t_f32(lay.m, lay.n, lay.seed)
    L, got, R = run_topk(hsl, W, "f32", "bf16", ATTN4096.frac)
    assert L.nnz() == 335_544
    ref = oracle.split_topk(W, ATTN4096.frac, "f32")
    refv = dict(ref)
    refv["val"] = ref_values(ref["val"], "f32", "bf16")
    check_csr_equal(got, refv, "bf16")
    assert np.array_equal(host(R).view(np.uint32), ref["R"].view(np.uint32))


@pytest.mark.parametrize("shape,frac,seed", [((2048, 1024), 0.05, 7), ((1000, 3000), 0.03, 8)])
def test_topk_bf16_single_pass(hsl, shape, frac, seed):
    W = synth.to_bf16_bits(synth.student_t_f32(*shape, seed))
    assert_topk_parity(hsl, W, "bf16", "bf16", frac)


# ---------------------------------------------------------------- top-k, ties and edges

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(300, 1000), (129, 77), (1, 5000), (4000, 1), (17, 8)])
@pytest.mark.parametrize("frac", [0.0, 1e-6, 0.031, 0.5, 1.0])
def test_topk_tie_heavy(hsl, dtype, shape, frac):
    W = tie_heavy(*shape, seed=shape[0] * 7 + shape[1], dtype=dtype)
    assert_topk_parity(hsl, W, dtype, dtype, frac)


@pytest.mark.parametrize("dtype,shape", [("bf16", (3, 40000)), ("f32", (5, 20000)),
                                         ("bf16", (70, 32768)), ("f32", (33, 16384))])
@pytest.mark.parametrize("frac", [0.01, 0.5])
def test_topk_wide_rows(hsl, dtype, shape, frac):
    """Rows wider than one 32 KB tile, and rows of exactly one tile."""
    W = tie_heavy(*shape, seed=shape[1], dtype=dtype)
    assert_topk_parity(hsl, W, dtype, dtype, frac)


@pytest.mark.parametrize("dtype,shape", [("bf16", (20000, 16)), ("bf16", (3000, 24)),
                                         ("f32", (5000, 12)), ("f32", (999, 8200))])
@pytest.mark.parametrize("frac", [0.05, 0.9])
def test_topk_tiles_across_many_rows(hsl, dtype, shape, frac):
    """Tiles that hold many short rows or start inside a row; at 0.9 a tile
    keeps more entries than it gathers in shared memory (the rest go straight
    to S)."""
    W = synth.as_storage(synth.student_t_f32(*shape, seed=shape[1]), dtype)
    assert_topk_parity(hsl, W, dtype, dtype, frac)


def test_topk_bf16_sampled_bracket_exact(hsl):
    """4M-element bf16 split: the threshold comes from the sampled bracket."""
    W = synth.to_bf16_bits(synth.student_t_f32(2048, 2048, seed=21))
    assert_topk_parity(hsl, W, "bf16", "bf16", 0.05)


def _sampled_positions(count):
    """Element indices the bf16 split samples (runs of 256 elements at a hashed
    offset in every stratum of 16384), restated here only to build an input
    whose sample misleads the bracket."""
    def mix32(x):
        x ^= x >> 16
        x = (x * 0x7FEB352D) & 0xFFFFFFFF
        x ^= x >> 15
        x = (x * 0x846CA68B) & 0xFFFFFFFF
        return x ^ (x >> 16)
    idx = []
    for c in range(count // 8 // 2048):
        v0 = c * 2048 + mix32(c) % (2048 - 32 + 1)
        idx.append(np.arange(v0 * 8, (v0 + 32) * 8))
    return np.concatenate(idx)


def test_topk_bf16_misleading_sample_falls_back(hsl):
    """Every sampled element is large and nothing else is: the bracket cannot
    hold the threshold, the full histogram pass runs, the split stays exact."""
    m, n = 2048, 2048
    W = synth.to_bf16_bits(synth.student_t_f32(m, n, seed=22) * np.float32(1e-3)).reshape(-1)
    W[_sampled_positions(m * n)] = 0x4700  # 32768.0
    assert_topk_parity(hsl, W.reshape(m, n), "bf16", "bf16", 0.05)


def test_topk_unaligned_input_pointer(hsl):
    """W and R starting 4 bytes past an allocation (scalar path)."""
    W = synth.student_t_f32(64, 130, 3)
    big = dev(np.concatenate([np.zeros(1, np.float32), W.reshape(-1)]), "f32")
    Wd = big[1:].view(64, 130)
    Rbig = torch.empty_like(big)
    R = Rbig[1:].view(64, 130)
    L = hsl.Layer(64, 130, 0, "csr", "f32")
    L.split(Wd, 0.1, R)
    got = L.get_sparse()
    ref = oracle.split_topk(W, 0.1, "f32")
    check_csr_equal(got, ref, "f32")
    assert np.array_equal(host(R).view(np.uint32), ref["R"].view(np.uint32))


def test_topk_nan_reported(hsl):
    W = synth.student_t_f32(40, 64, 1)
    W[3, 5] = np.nan
    L = hsl.Layer(40, 64, 0, "csr", "f32")
    L.split(dev(W, "f32"), 0.1, None)
    with pytest.raises(hsl.HslError) as e:
        L.check()
    assert e.value.name == "HSL_ERR_NAN_INPUT"
    L.check()   # cleared


def test_topk_repeat_calls_reuse(hsl):
    """Two splits in a row on one handle (look-back flags and tickets reset)."""
    W = synth.to_bf16_bits(synth.student_t_f32(512, 512, 4))
    L = hsl.Layer(512, 512, 0, "csr", "bf16")
    for frac in (0.05, 0.01, 0.05):
        L.split(dev(W, "bf16"), frac, None)
        got = L.get_sparse()
        ref = oracle.split_topk(W, frac, "bf16")
        check_csr_equal(got, ref, "bf16")


# ---------------------------------------------------------------- top-k at full size

def test_topk_70b_mlp_bf16_full_size_against_oracle(hsl):
    """28672×8192 bf16 at 5 % (11,744,051 kept): the GPU split against the
    oracle's full lexsort of all 234,881,024 entries, bit for bit (row_ptr,
    col, values, residual)."""
    lay = MLP70B.layers[0]
    W = synth.to_bf16_bits(synth.student_t_f32(lay.m, lay.n, lay.seed))
    L, got, R = run_topk(hsl, W, "bf16", "bf16", MLP70B.topk_frac_extra)
    assert L.nnz() == 11_744_051
    Rh = host(R)
    got_h = {"row_ptr": got["row_ptr"], "col": got["col"], "val": got["val"]}
    L.close()
    del R
    ref = oracle.split_topk(W, MLP70B.topk_frac_extra, "bf16")
    assert ref["k"] == 11_744_051
    check_csr_equal(got_h, ref, "bf16")
    assert np.array_equal(Rh.reshape(-1), ref["R"].reshape(-1)), "residual differs"


# ---------------------------------------------------------------- 2:4

def run_24(hsl, W_bits, w_dtype, layer_dtype):
    m, n = W_bits.shape
    L = hsl.Layer(m, n, 0, "nm24", layer_dtype)
    Wd = dev(W_bits, w_dtype)
    R = torch.empty_like(Wd)
    L.split(Wd, 0.5, R)
    L.check()
    got = L.get_sparse()
    torch.cuda.synchronize()
    return L, got, R


def assert_24_parity(hsl, W_bits, w_dtype, layer_dtype, rows=None):
    L, got, R = run_24(hsl, W_bits, w_dtype, layer_dtype)
    Wr = W_bits if rows is None else W_bits[rows]
    ref = oracle.split_24(np.ascontiguousarray(Wr), w_dtype)
    gv, gi, gR = host(got["val"]), got["idx"].cpu().numpy(), host(R)
    if rows is not None:
        gv, gi, gR = gv[rows], gi[rows], gR[rows]
    assert np.array_equal(gi, ref["idx"]), "indices differ"
    assert np.array_equal(as_bits(gv), as_bits(ref_values(ref["val"], w_dtype, layer_dtype))), \
        "values differ"
    assert np.array_equal(as_bits(gR), as_bits(ref["R"])), "residual differs"
    L.close()


def test_24_mlp_up_11008_bf16(hsl):
    lay = MLP_UP_11008.layers[0]
    W = synth.to_bf16_bits(synth.student_t_f32(lay.m, lay.n, lay.seed))
    assert_24_parity(hsl, W, "bf16", "bf16")


def test_24_mlp_70b_full_size_sampled_rows(hsl):
    lay = MLP70B.layers[0]
    W = synth.to_bf16_bits(synth.student_t_f32(lay.m, lay.n, lay.seed))
    rows = np.sort(np.random.default_rng(1).choice(lay.m, size=384, replace=False))
    rows[-1] = lay.m - 1
    assert_24_parity(hsl, W, "bf16", "bf16", rows)


@pytest.mark.parametrize("w_dtype,layer_dtype", [("f32", "f32"), ("f32", "bf16"), ("bf16", "f32")])
def test_24_dtype_mix(hsl, w_dtype, layer_dtype):
    W = synth.student_t_f32(96, 256, 5)
    W = W if w_dtype == "f32" else synth.to_bf16_bits(W)
    assert_24_parity(hsl, W, w_dtype, layer_dtype)


@pytest.mark.parametrize("shape", [(7, 12), (33, 20), (1, 4)])
def test_24_ties_and_odd_group_counts(hsl, shape):
    W = tie_heavy(*shape, seed=shape[0] + shape[1], dtype="bf16")
    assert_24_parity(hsl, W, "bf16", "bf16")
    Wf = tie_heavy(*shape, seed=shape[0] * 3, dtype="f32")
    assert_24_parity(hsl, Wf, "f32", "f32")


def test_24_nan_reported(hsl):
    W = synth.student_t_f32(8, 16, 2)
    W[1, 1] = np.nan
    L = hsl.Layer(8, 16, 0, "nm24", "f32")
    L.split(dev(W, "f32"), 0.5, None)
    with pytest.raises(hsl.HslError) as e:
        L.check()
    assert e.value.name == "HSL_ERR_NAN_INPUT"
