"""Float64 CPU oracle for the hierarchical sparse + low-rank (HSS) layer.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Nothing here is tuned;
every step is the plain definition, in the order the pages give it.

Sources (cited by page title and section):

* [HSS] "Hierarchical Sparse + Low-Rank Compression of LLMs"
  (LLMの階層的スパース+低ランク圧縮):
    - §Two-stage hierarchical sparse + low-rank compression: the decomposition
      W ≈ S + U Vᵀ with U ∈ R^{m×r}, V ∈ R^{n×r}; Stage 1 keeps the top 5 % of
      weights by absolute magnitude in a sparse (COO/CSR) matrix and leaves the
      rest as a dense residual; Stage 2 factors that residual into two
      1024×64 matrices; worked example 52,428 + 131,072 = 183,500 (5.7×).
    - §Implementation and operational patterns: the layer stores (S, U, V) and
      computes the forward pass as a sparse product plus two skinny dense
      products, never forming the full matrix.
* [HASSLE] HASSLE-free article (aibr.jp/archives/82335), §3 core technical
  elements: N:M structured sparsity as the GPU-friendly form of S.

Readings taken where the pages are silent or garbled (each one is listed in
the design notes as well):

1. Convention.  The page writes the forward in row-vector form
   ``output = input @ (S + U Vᵀ)``.  We use the column form y = Ŵ x with
   Ŵ ∈ R^{m×n} (m outputs, n inputs): X is [B, n], Y is [B, m], Y = X Ŵᵀ.
2. Top-k is global over the whole matrix, k = floor(frac · m · n) computed in
   IEEE double (the worked example's 5 % of 1,048,576 is 52,428).
3. Ties in |w| go to the lower linear index i·n + j.  In a 2:4 group ties go
   to the lower in-group index.
4. S stores the original values; the residual R is W with the selected
   positions set to +0.0 (bit pattern 0).
5. Ŵ = S + U Vᵀ everywhere (U Vᵀ is not masked at S positions).
6. -0.0 and +0.0 have equal magnitude; ±Inf is the largest magnitude; NaN is
   rejected; denormals are kept bit-exact.
7. The "recursive" low-rank stage is one truncated SVD, σ split as √σ on
   each side.

Pins (tests/test_oracle.py): the worked example's counts; O(N²) brute-force
ranking on 8×8 and 4-element groups with ties, ±0, ±Inf and denormals;
exact recovery of a planted S₀ + rank-r matrix; Eckart–Young; textbook CSR
SpMV (scipy) for r = 0; a pure-Python triple loop for the apply on tiny
shapes; the k = 0 and frac = 1 special cases.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "DTYPES", "bits_to_f64", "f32_to_bf16_bits", "topk_count", "magnitude",
    "split_topk", "split_24", "csr_to_dense", "nm24_to_dense",
    "lowrank_svd", "lowrank_randomized", "reconstruct", "apply",
    "apply_rows", "rel_err", "elem_rel_err", "param_counts", "nm24_count",
    "concentration", "rcm_order", "permute",
]

DTYPES = ("f32", "bf16")


# --------------------------------------------------------------------------
# Bit-level value handling.  Matrices are passed as their storage bits:
# float32 arrays for "f32", uint16 arrays holding bfloat16 bits for "bf16".
# --------------------------------------------------------------------------

def _as_bits(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        if a.dtype == np.float32:
            return a.view(np.uint32)
        if a.dtype == np.uint32:
            return a
    elif dtype == "bf16":
        if a.dtype == np.uint16:
            return a
    raise TypeError(f"array of {a.dtype} cannot hold {dtype} bits")


def bits_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of every stored element (f32 and bf16 both embed)."""
    b = _as_bits(a, dtype)
    if dtype == "f32":
        return b.view(np.float32).astype(np.float64)
    # a bf16 value is the upper half of the float32 with the same bits
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, round-to-nearest-even, returning uint16 bits.

    Written out on the integer bits: add 0x7FFF plus the lowest kept bit, then
    drop the low 16 bits.  NaN stays NaN (quiet bit forced); ±Inf stays ±Inf.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    is_nan = (u & 0x7FFFFFFF) > 0x7F800000
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) & 0xFFFF
    r = np.where(is_nan, ((u >> 16) | 0x40) & 0xFFFF, r)
    return r.astype(np.uint16)


# --------------------------------------------------------------------------
# Stage 1: magnitude split.
# --------------------------------------------------------------------------

def topk_count(frac: float, m: int, n: int) -> int:
    """k = floor(frac · m · n) in IEEE double; frac ≤ 0 → 0, frac ≥ 1 → m·n.

    [HSS] §Two-stage compression, worked example: 5 % of the 1,048,576
    entries of a 1024×1024 matrix is 52,428 (52,428.8 rounded down).
    """
    if frac != frac:
        raise ValueError("frac is NaN")
    total = m * n
    if frac <= 0.0:
        return 0
    if frac >= 1.0:
        return total
    return int(math.floor(frac * float(total)))


def magnitude(W: np.ndarray, dtype: str) -> np.ndarray:
    """|w| in float64 (exact for f32/bf16).  NaN is rejected (reading 6)."""
    v = bits_to_f64(W, dtype)
    if np.isnan(v).any():
        raise ValueError("NaN in W")
    return np.abs(v)


def split_topk(W: np.ndarray, frac: float, dtype: str) -> dict:
    """Stage 1, unstructured: keep the k largest |w| of the whole matrix.

    [HSS] §Two-stage compression: the top fraction of weights by absolute
    magnitude goes into a sparse matrix (COO or CSR); the remaining values
    form the dense residual.

    Done by a full sort, as the definition reads: order all m·n entries by
    (|w| descending, linear index ascending), take the first k.  Returns the
    canonical CSR of the selected set (row-major, columns ascending within a
    row) with the original value bits, and the residual bits.
    """
    m, n = W.shape
    bits = _as_bits(np.ascontiguousarray(W), dtype).reshape(-1)
    mag = magnitude(W, dtype).reshape(-1)
    k = topk_count(frac, m, n)
    lin = np.arange(m * n, dtype=np.int64)
    order = np.lexsort((lin, -mag))        # last key is primary
    chosen = np.sort(order[:k])            # row-major order of the kept set
    rows = chosen // n
    cols = chosen % n
    row_ptr = np.zeros(m + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(np.bincount(rows, minlength=m))
    resid = bits.copy()
    resid[chosen] = 0                      # +0.0 in either format
    return {
        "k": k,
        "row_ptr": row_ptr.astype(np.int32),
        "col": cols.astype(np.int32),
        "val": bits[chosen].copy(),
        "R": resid.reshape(m, n),
        "dtype": dtype,
    }


def nm24_count(m: int, n: int) -> int:
    """Number of values a 2:4 split keeps: two of every four inputs."""
    return m * (n // 4) * 2


def split_24(W: np.ndarray, dtype: str) -> dict:
    """Stage 1, 2:4 structured: in each row, in every group of four consecutive
    inputs, keep the two largest |w| (ties to the lower in-group index),
    stored in ascending column order.

    [HASSLE] §3: N:M sparsity is the structured form GPUs accelerate.

    Returns val [m, n/2] (value bits), idx [m, n/4] uint8 with the two kept
    in-group indices i0 < i1 packed as i0 | i1 << 2, and the residual bits.
    """
    m, n = W.shape
    if n % 4:
        raise ValueError("2:4 split needs n % 4 == 0")
    bits = _as_bits(np.ascontiguousarray(W), dtype).reshape(m, n // 4, 4)
    mag = magnitude(W, dtype).reshape(m, n // 4, 4)
    order = np.argsort(-mag, axis=2, kind="stable")   # stable: lower index first on ties
    kept = np.sort(order[:, :, :2], axis=2)
    val = np.take_along_axis(bits, kept, axis=2).reshape(m, n // 2)
    idx = (kept[:, :, 0] | (kept[:, :, 1] << 2)).astype(np.uint8)
    resid = bits.copy()
    np.put_along_axis(resid, kept, 0, axis=2)
    return {"val": val.copy(), "idx": idx, "R": resid.reshape(m, n), "dtype": dtype}


def csr_to_dense(m: int, n: int, row_ptr, col, val64) -> np.ndarray:
    """Dense float64 copy of a CSR matrix (duplicates, if any, add up)."""
    D = np.zeros((m, n), dtype=np.float64)
    rows = np.repeat(np.arange(m), np.diff(np.asarray(row_ptr, dtype=np.int64)))
    np.add.at(D, (rows, np.asarray(col, dtype=np.int64)), np.asarray(val64, dtype=np.float64))
    return D


def nm24_to_dense(val64: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Dense float64 copy of a 2:4 matrix from its values and in-group indices."""
    m, half = val64.shape
    n = half * 2
    g = n // 4
    D = np.zeros((m, g, 4), dtype=np.float64)
    v = val64.reshape(m, g, 2)
    i0 = (idx & 3).astype(np.int64)
    i1 = ((idx >> 2) & 3).astype(np.int64)
    np.put_along_axis(D, i0[:, :, None], v[:, :, 0:1], axis=2)
    np.put_along_axis(D, i1[:, :, None], v[:, :, 1:2], axis=2)
    return D.reshape(m, n)


# --------------------------------------------------------------------------
# Stage 2: low-rank factors of the residual (input preparation).
# --------------------------------------------------------------------------

def lowrank_svd(R64: np.ndarray, r: int) -> tuple[np.ndarray, np.ndarray]:
    """Truncated SVD of the residual: R ≈ U Vᵀ, U = U_r √Σ, V = V_r √Σ.

    [HSS] §Two-stage compression, Stage 2: the residual is factored into an
    m×r and an n×r matrix (1024×64 twice in the worked example).  One SVD is
    the reading of "recursive" taken here (reading 7).
    """
    m, n = R64.shape
    if r == 0:
        return np.zeros((m, 0)), np.zeros((n, 0))
    Uf, s, Vt = np.linalg.svd(R64, full_matrices=False)
    q = min(r, len(s))
    root = np.sqrt(s[:q])
    U = np.zeros((m, r))
    V = np.zeros((n, r))
    # a rank above min(m, n) is exact: the extra factor columns are zero
    U[:, :q] = Uf[:, :q] * root
    V[:, :q] = Vt[:q, :].T * root
    return U, V


def lowrank_randomized(R64: np.ndarray, r: int, omega: np.ndarray,
                       power_iters: int = 2) -> tuple[np.ndarray, np.ndarray]:
    """Randomised truncated SVD (Halko–Martinsson–Tropp range finder).

    ``omega`` is the n×(r+p) Gaussian test matrix, passed in so that the
    random draw is an input.  Steps: Y = R Ω; q power iterations
    Y ← R (Rᵀ Y) with re-orthonormalisation; Q = orth(Y); B = Qᵀ R;
    SVD of the small B; U = Q U_B √Σ, V = V_B √Σ truncated to r.
    """
    m, n = R64.shape
    if r == 0:
        return np.zeros((m, 0)), np.zeros((n, 0))
    Y = R64 @ omega
    Q, _ = np.linalg.qr(Y)
    for _ in range(power_iters):
        Z, _ = np.linalg.qr(R64.T @ Q)
        Q, _ = np.linalg.qr(R64 @ Z)
    Bm = Q.T @ R64
    Ub, s, Vt = np.linalg.svd(Bm, full_matrices=False)
    root = np.sqrt(s[:r])
    return (Q @ Ub[:, :r]) * root, Vt[:r, :].T * root


# --------------------------------------------------------------------------
# The forward pass.
# --------------------------------------------------------------------------

def reconstruct(S_dense64: np.ndarray, U64: np.ndarray, V64: np.ndarray) -> np.ndarray:
    """Ŵ = S + U Vᵀ in float64 ([HSS] §Two-stage compression, the equation)."""
    return S_dense64 + U64 @ V64.T


def apply(W_hat64: np.ndarray, X64: np.ndarray) -> np.ndarray:
    """Y = X Ŵᵀ: every token row x gives y = Ŵ x (column-form reading 1).

    [HSS] §Implementation and operational patterns: the layer's output is the
    input times (S + U Vᵀ).  The oracle forms Ŵ densely and multiplies, which
    is the plain definition; the split into S·x + U(Vᵀx) is what the kernels
    exploit and is not repeated here.
    """
    return np.asarray(X64, dtype=np.float64) @ W_hat64.T


def apply_rows(rows: np.ndarray, S_rows64: np.ndarray, U64: np.ndarray,
               V64: np.ndarray, X64: np.ndarray) -> np.ndarray:
    """Y[:, rows] for a sample of output rows: Ŵ[rows] = S[rows] + U[rows] Vᵀ.

    ``S_rows64`` is the dense float64 copy of just those rows of S.
    """
    W_rows = S_rows64 + U64[rows] @ V64.T
    return np.asarray(X64, dtype=np.float64) @ W_rows.T


def rel_err(Y: np.ndarray, Y_ref: np.ndarray) -> float:
    """max over tokens b of  max_i |Y_bi − Y*_bi| / max_i |Y*_bi|.

    A token whose reference row is all zero is compared absolutely.
    """
    Y = np.atleast_2d(np.asarray(Y, dtype=np.float64))
    R = np.atleast_2d(np.asarray(Y_ref, dtype=np.float64))
    if R.size == 0:
        return 0.0
    num = np.abs(Y - R).max(axis=1)
    den = np.abs(R).max(axis=1)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max())


def elem_rel_err(Y: np.ndarray, Y_ref: np.ndarray, floor: float = 1e-3) -> float:
    """max over tokens b and outputs i of
    |Y_bi − Y*_bi| / max(|Y*_bi|, floor · max_i |Y*_bi|).

    The element-wise companion of :func:`rel_err` (the target states a
    relative error without a norm; reading 11 reports both).  The floor keeps
    outputs that nearly cancel from dividing by ~0.  A token whose reference
    row is all zero is compared absolutely.
    """
    Y = np.atleast_2d(np.asarray(Y, dtype=np.float64))
    R = np.atleast_2d(np.asarray(Y_ref, dtype=np.float64))
    if R.size == 0:
        return 0.0
    rowmax = np.abs(R).max(axis=1, keepdims=True)
    den = np.maximum(np.abs(R), floor * rowmax)
    den = np.where(den > 0, den, 1.0)
    return float((np.abs(Y - R) / den).max())


# --------------------------------------------------------------------------
# Parameter accounting (the measurement the pages define).
# --------------------------------------------------------------------------

def param_counts(m: int, n: int, frac: float, r: int) -> dict:
    """Parameters of the compressed triple against the dense matrix.

    [HSS] §Two-stage compression, worked example, and §Measurement and
    validation (the parameter-reduction metric is compressed parameters over
    original parameters).
    """
    k = topk_count(frac, m, n)
    factor = r * (m + n)
    total = k + factor
    resid = m * n - k
    return {
        "dense": m * n,
        "sparse": k,
        "residual": resid,
        "factor": factor,
        "total": total,
        "reduction": (m * n) / total if total else math.inf,
        "residual_footprint_reduction": 1.0 - factor / resid if resid else 0.0,
    }


# --------------------------------------------------------------------------
# Permutation for concentration (a pre-processing step before Stage 1).
# --------------------------------------------------------------------------

def concentration(W: np.ndarray, dtype: str) -> float:
    """ρ = Σ_{(i,j) in the diagonal blocks} |W_ij| / Σ_{i,j} |W_ij|.

    [HSS] §Permutation and hierarchical alignment: the concentration ratio of
    the equation there, with "diagonal" the top-left and bottom-right blocks
    of the 2×2 block partition (the example names those two quadrants).
    Readings: the quadrants split at row ⌊m/2⌋ and column ⌊n/2⌋ (top-left =
    rows < ⌊m/2⌋ and columns < ⌊n/2⌋, bottom-right = the rest of both); an
    all-zero W has ρ = 0.
    """
    A = magnitude(W, dtype)
    m, n = A.shape
    mh, nh = m // 2, n // 2
    total = A.sum()
    if total == 0:
        return 0.0
    diag = A[:mh, :nh].sum() + A[mh:, nh:].sum()
    return float(diag / total)


def rcm_order(m: int, n: int, row_ptr, col) -> tuple[np.ndarray, np.ndarray]:
    """Reverse Cuthill–McKee order of the rows and columns of a sparse pattern.

    [HSS] §Permutation and hierarchical alignment: RCM reorders rows and
    columns so that the large entries gather near the diagonal (Cuthill &
    McKee's bandwidth-reducing ordering, reversed).  Reading for an m×n
    pattern: the graph is the bipartite row–column graph (vertex i < m is row
    i, vertex m + j is column j, an edge per stored entry), which needs no
    symmetric matrix; the order of its m + n vertices gives the row order and
    the column order.  The steps, in the classic form: take the unvisited
    vertex of smallest degree (ties: lowest vertex number) as the start of
    the next component; visit breadth first, appending each vertex's
    unvisited neighbours by increasing degree (ties: lowest vertex number);
    reverse the whole order at the end.

    Returns (row_order, col_order): row_order[k] is the original row placed
    k-th, col_order[k] the original column placed k-th.
    """
    rp = np.asarray(row_ptr, dtype=np.int64)
    cl = np.asarray(col, dtype=np.int64)
    V = m + n
    adj = [[] for _ in range(V)]
    for i in range(m):
        for j in cl[rp[i]:rp[i + 1]]:
            adj[i].append(m + int(j))
            adj[m + int(j)].append(i)
    deg = [len(a) for a in adj]
    visited = [False] * V
    order = []
    by_degree = sorted(range(V), key=lambda v: (deg[v], v))
    for start in by_degree:
        if visited[start]:
            continue
        visited[start] = True
        queue = [start]
        head = 0
        while head < len(queue):
            v = queue[head]
            head += 1
            fresh = sorted({u for u in adj[v] if not visited[u]}, key=lambda u: (deg[u], u))
            for u in fresh:
                visited[u] = True
                queue.append(u)
        order.extend(queue)
    order.reverse()
    rows = np.array([v for v in order if v < m], dtype=np.int32)
    cols = np.array([v - m for v in order if v >= m], dtype=np.int32)
    return rows, cols


def permute(W: np.ndarray, row_order, col_order) -> np.ndarray:
    """W' with W'[k, l] = W[row_order[k], col_order[l]] (bits copied)."""
    return np.ascontiguousarray(np.asarray(W)[np.asarray(row_order)][:, np.asarray(col_order)])
