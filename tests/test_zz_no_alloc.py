"""hsl_split_topk_noalloc, the split for callers that cannot allocate device
memory (a serving runtime or plugin host that owns every byte, code that must
not synchronise the device through cudaMalloc/cudaFree).  It keeps its
scratch in a fixed static device array, so these tests check that, called
twice in a row through the C ABI, it returns exactly what the handle-based
hsl_split_topk returns and exactly what the float64 oracle's full-sort split
returns (the split's tolerance is bit-exactness), and that it refuses sizes
its array cannot hold and a missing status word.

The file name sorts last so that a run stopping at the first failure has run
every other test before this one."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import ref_values
from sparse_rank_linear_03_b200 import hsl, synth

pytestmark = pytest.mark.gpu

DT = {"f32": 0, "bf16": 1}


def _bits(t):
    return synth.storage_from_torch(t).view(np.uint16 if t.dtype == torch.bfloat16 else np.uint32)


def _noalloc(W, m, n, w_dtype, frac, val_dtype):
    k = int(math.floor(frac * m * n)) if 0 < frac < 1 else (0 if frac <= 0 else m * n)
    dev = W.device
    rp = torch.full((m + 1,), -1, dtype=torch.int32, device=dev)
    col = torch.full((max(k, 1),), -1, dtype=torch.int32, device=dev)
    val = torch.zeros(max(k, 1), dtype=hsl.TORCH_DTYPE[val_dtype], device=dev)
    R = torch.empty_like(W)
    status = torch.full((1,), 7, dtype=torch.int32, device=dev)
    st = hsl.lib.hsl_split_topk_noalloc(
        W.data_ptr(), m, n, DT[w_dtype], frac, rp.data_ptr(), col.data_ptr(), val.data_ptr(),
        DT[val_dtype], R.data_ptr(), status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, hsl.lib.hsl_last_message()
    torch.cuda.synchronize()
    return rp, col[:k], val[:k], R, int(status.item())


@pytest.mark.parametrize("case", [0, 1])
def test_noalloc_split_matches_handle_split_on_two_calls(case):
    runs = [  # (m, n, frac, W dtype, value dtype, seed): two different calls in a row
        [(1024, 1024, 0.05, "f32", "f32", 0), (777, 3000, 0.03, "bf16", "bf16", 1)],
        [(4096, 4096, 0.02, "f32", "bf16", 2000), (300, 50000, 0.01, "bf16", "bf16", 3)],
    ][case]
    for m, n, frac, wdt, vdt, seed in runs:
        Wf = synth.student_t_f32(m, n, seed)
        W = synth.torch_from_storage(synth.as_storage(Wf, wdt), wdt, "cuda")
        rp, col, val, R, status = _noalloc(W, m, n, wdt, frac, vdt)
        L = hsl.Layer(m, n, 0, "csr", vdt)
        Rref = torch.empty_like(W)
        L.split(W, frac, Rref)
        ref = L.get_sparse()
        torch.cuda.synchronize()
        assert status == 0
        assert torch.equal(rp, ref["row_ptr"])
        assert torch.equal(col, ref["col"])
        assert np.array_equal(_bits(val), _bits(ref["val"]))
        assert np.array_equal(_bits(R), _bits(Rref))
        L.close()
        # and against the oracle's full sort, bit for bit
        Wbits = synth.as_storage(Wf, wdt)
        o = oracle.split_topk(Wbits, frac, wdt)
        assert np.array_equal(rp.cpu().numpy(), o["row_ptr"])
        assert np.array_equal(col.cpu().numpy(), o["col"])
        want = ref_values(o["val"], wdt, vdt)
        assert np.array_equal(_bits(val), want.view(np.uint16 if vdt == "bf16" else np.uint32))
        assert np.array_equal(_bits(R).reshape(-1),
                              o["R"].reshape(-1).view(np.uint16 if wdt == "bf16" else np.uint32))


def test_noalloc_split_refuses_sizes_beyond_its_scratch():
    W = torch.zeros(1, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    p, sp = W.data_ptr(), status.data_ptr()
    big_m = ctypes.c_int64(65537)
    st = hsl.lib.hsl_split_topk_noalloc(p, big_m, 4, 0, 0.5, p, p, p, 0, None, sp, None)
    assert hsl.STATUS[st] == "HSL_ERR_UNSUPPORTED"
    assert b"65536" in hsl.lib.hsl_last_message()
    # a huge n is refused before m·n is formed (2 · 2^62 would overflow int64)
    st = hsl.lib.hsl_split_topk_noalloc(p, 2, ctypes.c_int64(1 << 62), 0, 0.5, p, p, p, 0, None,
                                        sp, None)
    assert hsl.STATUS[st] == "HSL_ERR_UNSUPPORTED"
    st = hsl.lib.hsl_split_topk_noalloc(p, 3, ctypes.c_int64((1 << 31) - 1), 0, 0.5, p, p, p, 0,
                                        None, sp, None)
    assert hsl.STATUS[st] == "HSL_ERR_UNSUPPORTED"


def test_noalloc_split_needs_a_status_word():
    """Without the status word a NaN in W or a wait that gave up would go
    unreported, so the call refuses a NULL one."""
    W = torch.zeros(4, 4, dtype=torch.float32, device="cuda")
    rp = torch.zeros(5, dtype=torch.int32, device="cuda")
    st = hsl.lib.hsl_split_topk_noalloc(W.data_ptr(), 4, 4, 0, 0.0, rp.data_ptr(), None, None, 0,
                                        None, None, None)
    assert hsl.STATUS[st] == "HSL_ERR_INVALID_ARG"
    assert b"status" in hsl.lib.hsl_last_message()
