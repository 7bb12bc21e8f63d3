"""ctypes binding of libhsl (include/hsl.h).

Argument marshalling only: every step of the split, pack and apply runs in
libhsl's CUDA kernels.  torch tensors supply device memory and the current
stream.  Importing this module loads ``libhsl.so`` and raises ImportError if
it has not been built (``python -m sparse_rank_linear_03_b200.build``); there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhsl.so")

FMT = {"csr": 0, "nm24": 1}
DTYPE = {"f32": 0, "bf16": 1}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}
STATUS = {0: "HSL_OK", 1: "HSL_ERR_INVALID_ARG", 2: "HSL_ERR_UNSUPPORTED", 3: "HSL_ERR_NOT_READY",
          4: "HSL_ERR_OOM", 5: "HSL_ERR_CUDA", 6: "HSL_ERR_NAN_INPUT", 7: "HSL_ERR_TIMEOUT"}

# every symbol include/hsl.h declares
EXPORTS = (
    "hsl_create", "hsl_destroy", "hsl_split_topk", "hsl_get_nnz", "hsl_get_sparse",
    "hsl_set_sparse_csr", "hsl_set_sparse_nm24", "hsl_pack", "hsl_apply",
    "hsl_group_create", "hsl_group_apply", "hsl_group_destroy", "hsl_check",
    "hsl_status_str", "hsl_last_message", "hsl_launch_count", "hsl_split_topk_noalloc",
    "hsl_concentration", "hsl_rcm_order", "hsl_permute", "hsl_set_permutation", "hsl_factor",
    "hsl_set_index_bits",
)


class HslError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name}: {message}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_rank_linear_03_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    sig = {
        "hsl_create": [I64, I64, I32, ctypes.c_int, ctypes.c_int, ctypes.POINTER(P)],
        "hsl_destroy": [P],
        "hsl_split_topk": [P, P, ctypes.c_int, D, P, P],
        "hsl_get_nnz": [P, ctypes.POINTER(I64)],
        "hsl_get_sparse": [P, P, P, P, P, P],
        "hsl_set_sparse_csr": [P, I64, P, P, P, P],
        "hsl_set_sparse_nm24": [P, P, P, P],
        "hsl_pack": [P, P, P, P],
        "hsl_apply": [P, P, P, I64, P],
        "hsl_group_create": [P, I32, ctypes.POINTER(P), P],
        "hsl_group_apply": [P, P, P, I64, P],
        "hsl_group_destroy": [P],
        "hsl_check": [P, P],
        "hsl_status_str": [ctypes.c_int],
        "hsl_last_message": [],
        "hsl_launch_count": [],
        "hsl_split_topk_noalloc": [P, I64, I64, ctypes.c_int, D, P, P, P, ctypes.c_int, P, P, P],
        "hsl_concentration": [P, I64, I64, ctypes.c_int, ctypes.POINTER(D), P],
        "hsl_rcm_order": [I64, I64, P, P, P, P],
        "hsl_permute": [P, I64, I64, ctypes.c_int, P, P, P, P],
        "hsl_set_permutation": [P, P, P, P],
        "hsl_factor": [P, P, ctypes.c_int, P, I32, I32, P, P, P, P],
        "hsl_set_index_bits": [P, I32],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.hsl_status_str.restype = ctypes.c_char_p
    lib.hsl_last_message.restype = ctypes.c_char_p
    lib.hsl_launch_count.restype = ctypes.c_uint64
    return lib


lib = _load()


def _ok(status: int, where: str) -> None:
    if status != 0:
        raise HslError(status, where, lib.hsl_last_message().decode(errors="replace"))


def _stream(stream) -> int:
    if stream is not None:
        return int(getattr(stream, "cuda_stream", stream))
    return torch.cuda.current_stream().cuda_stream


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return t.data_ptr()
    return int(t)


def _need(t, numel: int, what: str) -> None:
    if t is not None and isinstance(t, torch.Tensor) and t.numel() != numel:
        raise ValueError(f"{what} has {t.numel()} elements, expected {numel}")


def _dtype_of(t, want: str, what: str) -> None:
    if isinstance(t, torch.Tensor) and t.dtype != TORCH_DTYPE[want]:
        raise ValueError(f"{what} is {t.dtype}, the layer stores {want}")


def _wdtype(t: torch.Tensor) -> str:
    return {torch.float32: "f32", torch.bfloat16: "bf16"}[t.dtype]


def concentration(W: torch.Tensor, stream=None) -> float:
    """ρ of a device matrix W (hsl_concentration)."""
    m, n = W.shape
    rho = ctypes.c_double()
    _ok(lib.hsl_concentration(_ptr(W), m, n, DTYPE[_wdtype(W)], ctypes.byref(rho), _stream(stream)),
        "hsl_concentration")
    return rho.value


def rcm_order(m: int, n: int, row_ptr, col):
    """RCM row and column orders of a CSR pattern (hsl_rcm_order; host arrays)."""
    import numpy as np
    rp = np.ascontiguousarray(np.asarray(row_ptr, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(col, dtype=np.int32))
    ro = np.empty(m, np.int32)
    co = np.empty(n, np.int32)
    _ok(lib.hsl_rcm_order(m, n, rp.ctypes.data, cl.ctypes.data if cl.size else None,
                          ro.ctypes.data, co.ctypes.data), "hsl_rcm_order")
    return ro, co


def permute(W: torch.Tensor, row_order: torch.Tensor, col_order: torch.Tensor,
            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[k][l] = W[row_order[k]][col_order[l]] on the device (hsl_permute)."""
    m, n = W.shape
    _need(row_order, m, "row_order")
    _need(col_order, n, "col_order")
    if out is None:
        out = torch.empty_like(W)
    _ok(lib.hsl_permute(_ptr(W), m, n, DTYPE[_wdtype(W)], _ptr(row_order), _ptr(col_order),
                        _ptr(out), _stream(stream)), "hsl_permute")
    return out


def launch_count() -> int:
    """Kernels libhsl has launched in this process."""
    return int(lib.hsl_launch_count())


class Layer:
    """One compressed layer: W ≈ S + U Vᵀ held on the device (an hsl_handle)."""

    def __init__(self, m: int, n: int, r: int, fmt: str = "csr", dtype: str = "bf16"):
        self.m, self.n, self.r, self.fmt, self.dtype = m, n, r, fmt, dtype
        h = ctypes.c_void_p()
        _ok(lib.hsl_create(m, n, r, FMT[fmt], DTYPE[dtype], ctypes.byref(h)), "hsl_create")
        self._h = h

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            lib.hsl_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- stage 1 ------------------------------------------------------------
    def split(self, W: torch.Tensor, frac: float, residual: torch.Tensor | None = None,
              stream=None) -> None:
        wdt = {torch.float32: "f32", torch.bfloat16: "bf16"}[W.dtype]
        _need(W, self.m * self.n, "W")
        if residual is not None and (residual.dtype != W.dtype or residual.numel() != W.numel()):
            raise ValueError("residual must match W")
        _ok(lib.hsl_split_topk(self._h, _ptr(W), DTYPE[wdt], float(frac), _ptr(residual),
                               _stream(stream)), "hsl_split_topk")

    def nnz(self) -> int:
        v = ctypes.c_int64()
        _ok(lib.hsl_get_nnz(self._h, ctypes.byref(v)), "hsl_get_nnz")
        return v.value

    def get_sparse(self, stream=None) -> dict:
        dev = torch.device("cuda")
        vt = TORCH_DTYPE[self.dtype]
        if self.fmt == "csr":
            k = self.nnz()
            rp = torch.empty(self.m + 1, dtype=torch.int32, device=dev)
            col = torch.empty(max(k, 1), dtype=torch.int32, device=dev)
            val = torch.empty(max(k, 1), dtype=vt, device=dev)
            _ok(lib.hsl_get_sparse(self._h, _ptr(rp), _ptr(col), _ptr(val), None, _stream(stream)),
                "hsl_get_sparse")
            return {"row_ptr": rp, "col": col[:k], "val": val[:k]}
        val = torch.empty(self.m, self.n // 2, dtype=vt, device=dev)
        idx = torch.empty(self.m, self.n // 4, dtype=torch.uint8, device=dev)
        _ok(lib.hsl_get_sparse(self._h, None, None, _ptr(val), _ptr(idx), _stream(stream)),
            "hsl_get_sparse")
        return {"val": val, "idx": idx}

    def set_sparse_csr(self, row_ptr, col, val, stream=None) -> None:
        _need(row_ptr, self.m + 1, "row_ptr")
        _need(val, col.numel(), "val")
        _dtype_of(val, self.dtype, "val")
        _ok(lib.hsl_set_sparse_csr(self._h, int(col.numel()), _ptr(row_ptr), _ptr(col), _ptr(val),
                                   _stream(stream)), "hsl_set_sparse_csr")

    def set_sparse_nm24(self, val, idx, stream=None) -> None:
        _need(val, self.m * (self.n // 2), "val")
        _need(idx, self.m * (self.n // 4), "idx")
        _dtype_of(val, self.dtype, "val")
        _ok(lib.hsl_set_sparse_nm24(self._h, _ptr(val), _ptr(idx), _stream(stream)),
            "hsl_set_sparse_nm24")

    def set_index_bits(self, bits: int) -> None:
        """Column width of the packed CSR S (8, 16, 32; 0 = default) from the next pack."""
        _ok(lib.hsl_set_index_bits(self._h, int(bits)), "hsl_set_index_bits")

    # -- pack + apply -------------------------------------------------------
    def pack(self, U, V, stream=None) -> None:
        _need(U, self.m * self.r, "U")
        _need(V, self.n * self.r, "V")
        _dtype_of(U, self.dtype, "U")
        _dtype_of(V, self.dtype, "V")
        _ok(lib.hsl_pack(self._h, _ptr(U), _ptr(V), _stream(stream)), "hsl_pack")

    def apply(self, X: torch.Tensor, Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        batch = X.shape[0] if X.dim() == 2 else 1
        _need(X, batch * self.n, "X")
        _dtype_of(X, self.dtype, "X")
        if Y is not None:
            _need(Y, batch * self.m, "Y")
            _dtype_of(Y, self.dtype, "Y")
        if Y is None:
            Y = torch.empty(batch, self.m, dtype=X.dtype, device=X.device,
                            pin_memory=(X.device.type == "cpu"))
        _ok(lib.hsl_apply(self._h, _ptr(X), _ptr(Y), batch, _stream(stream)), "hsl_apply")
        return Y

    def factor(self, R: torch.Tensor, omega: torch.Tensor, power_iters: int = 2, stream=None):
        """Stage 2: U [m][r], V [n][r] (layer dtype) and σ [r] of the residual R
        by the randomized truncated SVD with test matrix omega [n][k] (fp32)."""
        _need(R, self.m * self.n, "R")
        if omega.dtype != torch.float32 or omega.dim() != 2 or omega.shape[0] != self.n:
            raise ValueError("omega must be fp32 [n][k]")
        dev = R.device
        U = torch.empty(self.m, self.r, dtype=TORCH_DTYPE[self.dtype], device=dev)
        V = torch.empty(self.n, self.r, dtype=TORCH_DTYPE[self.dtype], device=dev)
        sig = torch.empty(self.r, dtype=torch.float32, device=dev)
        _ok(lib.hsl_factor(self._h, _ptr(R), DTYPE[_wdtype(R)], _ptr(omega), int(omega.shape[1]),
                           int(power_iters), _ptr(U), _ptr(V), _ptr(sig), _stream(stream)),
            "hsl_factor")
        return U, V, sig

    def set_permutation(self, row_order, col_order, stream=None) -> None:
        """The layer holds W[row_order][:, col_order]; apply in the original order."""
        if row_order is not None:
            _need(row_order, self.m, "row_order")
            _need(col_order, self.n, "col_order")
        _ok(lib.hsl_set_permutation(self._h, _ptr(row_order), _ptr(col_order), _stream(stream)),
            "hsl_set_permutation")

    def check(self, stream=None) -> None:
        _ok(lib.hsl_check(self._h, _stream(stream)), "hsl_check")


class Group:
    """Several packed layers applied in one pass (hsl_group)."""

    def __init__(self, layers: list[Layer], stream=None):
        self.layers = list(layers)
        arr = (ctypes.c_void_p * len(layers))(*[l.handle.value for l in layers])
        g = ctypes.c_void_p()
        _ok(lib.hsl_group_create(arr, len(layers), ctypes.byref(g), _stream(stream)),
            "hsl_group_create")
        self._g = g
        self._tabs = None

    def apply(self, Xs: list[torch.Tensor], Ys: list[torch.Tensor], stream=None) -> None:
        batch = Xs[0].shape[0]
        if len(Xs) != len(self.layers) or len(Ys) != len(self.layers):
            raise ValueError("one X and one Y per layer")
        for l, x, y in zip(self.layers, Xs, Ys):
            _need(x, batch * l.n, "X")
            _need(y, batch * l.m, "Y")
        xa = (ctypes.c_void_p * len(Xs))(*[_ptr(x) for x in Xs])
        ya = (ctypes.c_void_p * len(Ys))(*[_ptr(y) for y in Ys])
        _ok(lib.hsl_group_apply(self._g, xa, ya, batch, _stream(stream)), "hsl_group_apply")

    def close(self) -> None:
        if getattr(self, "_g", None) is not None and self._g.value:
            lib.hsl_group_destroy(self._g)
            self._g = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
