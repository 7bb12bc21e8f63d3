"""C-ABI tests that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host with the documented
status codes (no device call is reached on these paths)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hsl.h")

hsl = pytest.importorskip("sparse_rank_linear_03_b200.hsl")
lib = hsl.lib

OK, INVALID, UNSUPPORTED, NOT_READY, OOM = 0, 1, 2, 3, 4


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hsl_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(hsl.EXPORTS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", hsl.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (hsl_\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_is_built_for_sm100a():
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", hsl.LIB_PATH],
                         capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    assert "sm_100a" in out.stdout


def _create(m=8, n=8, r=2, fmt=0, dt=0):
    h = ctypes.c_void_p()
    st = lib.hsl_create(m, n, r, fmt, dt, ctypes.byref(h))
    return st, h


def test_status_strings():
    for code in range(8):
        assert lib.hsl_status_str(code)
    assert lib.hsl_status_str(99) == b"unknown status"


@pytest.mark.parametrize("args,code", [
    ((0, 8, 2, 0, 0), INVALID),
    ((8, 0, 2, 0, 0), INVALID),
    ((8, 8, -1, 0, 0), UNSUPPORTED),
    ((8, 8, 257, 0, 0), UNSUPPORTED),
    ((8, 8, 2, 7, 0), INVALID),
    ((8, 8, 2, 0, 9), INVALID),
    ((8, 6, 2, 1, 0), UNSUPPORTED),          # 2:4 needs n % 4 == 0
    ((1 << 16, 1 << 15, 2, 0, 0), UNSUPPORTED),  # m*n >= 2^31
])
def test_create_rejects(args, code):
    h = ctypes.c_void_p()
    assert lib.hsl_create(*args, ctypes.byref(h)) == code
    assert not h.value
    assert lib.hsl_last_message()


def test_create_null_out():
    assert lib.hsl_create(8, 8, 2, 0, 0, None) == INVALID


def test_host_side_checks_before_any_device_call():
    st, h = _create()
    assert st == OK and h.value
    try:
        assert lib.hsl_split_topk(h, None, 0, 0.5, None, None) == INVALID        # W NULL
        assert lib.hsl_split_topk(h, 16, 5, 0.5, None, None) == INVALID          # bad dtype
        assert lib.hsl_split_topk(h, 16, 0, float("nan"), None, None) == INVALID
        assert lib.hsl_pack(h, None, None, None) == INVALID                      # r > 0, U NULL
        assert lib.hsl_pack(h, 16, 16, None) == NOT_READY                        # no S yet
        assert lib.hsl_apply(h, 16, 16, 1, None) == NOT_READY                    # not packed
        assert lib.hsl_apply(h, 16, 16, -1, None) == INVALID
        assert lib.hsl_apply(h, 16, 16, 0, None) == OK                           # batch 0: no-op
        assert lib.hsl_apply(h, None, 16, 1, None) == INVALID
        assert lib.hsl_get_sparse(h, None, None, None, None, None) == NOT_READY
        assert lib.hsl_set_sparse_nm24(h, 16, 16, None) == INVALID               # CSR handle
        assert lib.hsl_set_sparse_csr(h, -1, 16, 16, 16, None) == INVALID
        assert lib.hsl_set_sparse_csr(h, 65, 16, 16, 16, None) == INVALID        # nnz > m*n
        nnz = ctypes.c_int64(-1)
        assert lib.hsl_get_nnz(h, ctypes.byref(nnz)) == OK and nnz.value == 0
        assert lib.hsl_get_nnz(h, None) == INVALID
        assert lib.hsl_check(h, None) == OK                                      # nothing recorded
    finally:
        assert lib.hsl_destroy(h) == OK


def test_nm24_handle_checks():
    st, h = _create(8, 16, 4, 1, 1)
    assert st == OK
    try:
        assert lib.hsl_split_topk(h, 16, 1, 0.3, None, None) == UNSUPPORTED      # frac != 0.5
        assert lib.hsl_set_sparse_csr(h, 1, 16, 16, 16, None) == INVALID         # not CSR
        assert lib.hsl_set_sparse_nm24(h, None, 16, None) == INVALID
    finally:
        lib.hsl_destroy(h)


def test_null_handles_and_groups():
    assert lib.hsl_destroy(None) == OK
    assert lib.hsl_group_destroy(None) == OK
    assert lib.hsl_split_topk(None, 16, 0, 0.5, None, None) == INVALID
    assert lib.hsl_apply(None, 16, 16, 1, None) == INVALID
    assert lib.hsl_check(None, None) == INVALID
    g = ctypes.c_void_p()
    assert lib.hsl_group_create(None, 0, ctypes.byref(g), None) == INVALID
    st, h = _create()
    arr = (ctypes.c_void_p * 1)(h.value)
    assert lib.hsl_group_create(arr, 1, ctypes.byref(g), None) == NOT_READY    # not packed
    assert lib.hsl_group_apply(None, None, None, 1, None) == INVALID
    lib.hsl_destroy(h)


def test_fault_injection_alloc_reports_oom(monkeypatch):
    """Host-side failure path: the first allocation fails, nothing is launched."""
    monkeypatch.setenv("HSL_FAULT_INJECT", "alloc")
    st, h = _create()
    try:
        before = lib.hsl_launch_count()
        assert lib.hsl_split_topk(h, 16, 0, 0.5, None, None) == OOM
        assert b"HSL_FAULT_INJECT" in lib.hsl_last_message()
        assert lib.hsl_launch_count() == before
    finally:
        lib.hsl_destroy(h)


def test_binding_raises_typed_errors():
    with pytest.raises(hsl.HslError) as e:
        hsl.Layer(0, 4, 1)
    assert e.value.name == "HSL_ERR_INVALID_ARG"


# ---------------------------------------------------------------- the later entry points

def test_index_bits_checks():
    st, h = _create(8, 8, 2, 0, 1)
    assert st == OK
    assert lib.hsl_set_index_bits(h, 12) == INVALID
    for bits in (0, 8, 16, 32):
        assert lib.hsl_set_index_bits(h, bits) == OK
    lib.hsl_destroy(h)
    st, h = _create(8, 8, 2, 1, 1)       # 2:4 handle
    assert lib.hsl_set_index_bits(h, 8) == UNSUPPORTED
    lib.hsl_destroy(h)
    st, h = _create(4, 70000, 2, 0, 1)   # n ≥ 65535: only 32-bit columns
    assert lib.hsl_set_index_bits(h, 16) == UNSUPPORTED
    assert lib.hsl_set_index_bits(h, 8) == UNSUPPORTED
    assert lib.hsl_set_index_bits(h, 32) == OK
    lib.hsl_destroy(h)


def test_factor_checks_before_any_device_work():
    st, h = _create(64, 32, 8, 0, 0)
    p = ctypes.c_void_p(16)
    assert lib.hsl_factor(h, None, 0, p, 16, 1, p, p, p, None) == INVALID
    assert lib.hsl_factor(h, p, 0, p, 4, 1, p, p, p, None) == UNSUPPORTED       # k < r
    assert lib.hsl_factor(h, p, 0, p, 40, 1, p, p, p, None) == UNSUPPORTED      # k > min(m, n)
    assert lib.hsl_factor(h, p, 0, p, 16, -1, p, p, p, None) == INVALID
    assert lib.hsl_factor(h, p, 0, p, 16, 1, None, p, p, None) == INVALID
    lib.hsl_destroy(h)


def test_permutation_calls_check_arguments_on_the_host():
    rho = ctypes.c_double()
    assert lib.hsl_concentration(None, 4, 4, 0, ctypes.byref(rho), None) == INVALID
    assert lib.hsl_concentration(ctypes.c_void_p(16), 0, 4, 0, ctypes.byref(rho), None) == INVALID
    p = ctypes.c_void_p(16)
    assert lib.hsl_permute(p, 4, 4, 5, p, p, p, None) == INVALID
    assert lib.hsl_set_permutation(None, p, p, None) == INVALID
    st, h = _create(8, 8, 2, 0, 0)
    assert lib.hsl_set_permutation(h, p, None, None) == INVALID   # one order without the other
    assert lib.hsl_set_permutation(h, None, None, None) == OK     # clearing needs no device
    lib.hsl_destroy(h)


def _rcm(m, n, rp, col):
    import numpy as np
    rp = np.ascontiguousarray(rp, dtype=np.int32)
    col = np.ascontiguousarray(col, dtype=np.int32)
    ro = np.empty(m, np.int32)
    co = np.empty(n, np.int32)
    st = lib.hsl_rcm_order(m, n, rp.ctypes.data, col.ctypes.data if col.size else None,
                           ro.ctypes.data, co.ctypes.data)
    return st, ro, co


def test_rcm_order_is_the_oracles_on_random_patterns():
    """The RCM order is a host-side graph step of the library: identical to the
    oracle's on random patterns, empty rows and columns included."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(0)
    for _ in range(60):
        m, n = int(rng.integers(1, 70)), int(rng.integers(1, 70))
        mask = rng.random((m, n)) < rng.uniform(0.0, 0.2)
        rp = np.zeros(m + 1, np.int64)
        rp[1:] = np.cumsum(mask.sum(1))
        col = np.nonzero(mask)[1]
        st, ro, co = _rcm(m, n, rp, col)
        assert st == OK
        wr, wc = oracle.rcm_order(m, n, rp, col)
        assert np.array_equal(ro, wr) and np.array_equal(co, wc)


def test_rcm_order_rejects_bad_patterns():
    import numpy as np
    assert _rcm(3, 4, [1, 1, 2, 2], [0, 1])[0] == INVALID          # row_ptr[0] != 0
    assert _rcm(3, 4, [0, 2, 1, 2], [0, 1])[0] == INVALID          # not monotone
    assert _rcm(2, 4, [0, 1, 2], [0, 9])[0] == INVALID             # column outside [0, n)
    assert _rcm(2, 2, [0, 1, 9], np.zeros(9, np.int32))[0] == INVALID  # more entries than m·n
