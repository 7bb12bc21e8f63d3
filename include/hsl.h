/*
 * hsl.h — C ABI of libhsl: weight matrices compressed as W ≈ S + U Vᵀ
 * ("hierarchical sparse + low-rank"), split and applied on one B200 (sm_100a).
 *
 * Source of the operations (cited by page title and section):
 *   [HSS]    "Hierarchical Sparse + Low-Rank Compression of LLMs"
 *            (LLMの階層的スパース+低ランク圧縮)
 *            - §Two-stage hierarchical sparse + low-rank compression:
 *              W ≈ S + U Vᵀ, U ∈ R^{m×r}, V ∈ R^{n×r}; Stage 1 keeps the
 *              largest-magnitude weights in a sparse matrix (COO/CSR), the
 *              rest is the dense residual; Stage 2 factors the residual.
 *            - §Implementation and operational patterns: the layer holds
 *              (S, U, V) and computes the forward as a sparse product plus
 *              two small dense products without forming W.
 *            - §Implementation and operational patterns (from theory to
 *              production), mixed precision: 16-bit factors and narrow
 *              sparse indices.
 *   [HASSLE] HASSLE-free article (aibr.jp/archives/82335), §3: N:M
 *            structured sparsity as the GPU-friendly form of S.
 *   [SQZ]    SqueezeLLM article (aibr.jp/archives/208940), §1: single-batch
 *            decoding is bound by reading the weights from memory.
 *
 * Conventions (all entry points):
 *   - Shapes: W and Ŵ are m×n (m output features, n input features),
 *     row-major.  X is [batch][n], Y is [batch][m], row-major, and each row
 *     satisfies y = Ŵ x = S x + U (Vᵀ x).  (The page writes the same product
 *     in row-vector form, output = input @ (S + U Vᵀ); this is its transpose.)
 *   - Data pointers are DEVICE pointers owned by the caller, unless an entry
 *     point says otherwise.  The handle owns only its own copies (canonical
 *     and packed S, U, V) and workspace, allocated by the call that first
 *     needs them and released by hsl_destroy.
 *   - Every call taking a stream is asynchronous and stream-ordered on it.
 *     A stream is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Host-side argument checks return immediately; launch errors
 *     come back as HSL_ERR_CUDA.  Errors found on the device (NaN in W, a
 *     bounded wait that ran out) are recorded in the handle and returned by
 *     hsl_check.  Nothing aborts and no C++ exception crosses the ABI.
 *   - A handle is not thread-safe and keeps per-call workspace: use one
 *     handle per stream, and do not overlap calls on one handle across
 *     streams.
 *   - hsl_check reports a CSR column index outside [0, n) found while packing
 *     an imported S as HSL_ERR_INVALID_ARG (the entry is dropped).
 *   - Calls that allocate (the first split/set/pack/apply of a handle, or a
 *     split with a larger k than before) must not be made under stream
 *     capture; repeat calls with the same sizes allocate nothing.
 */
#ifndef HSL_H_
#define HSL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct hsl_handle_s* hsl_handle;
typedef void* hsl_stream; /* cudaStream_t */

typedef enum {
  HSL_OK = 0,
  HSL_ERR_INVALID_ARG = 1, /* a NULL/out-of-range argument, host-side check */
  HSL_ERR_UNSUPPORTED = 2, /* a valid request the library does not handle   */
  HSL_ERR_NOT_READY = 3,   /* e.g. hsl_apply before hsl_pack                */
  HSL_ERR_OOM = 4,         /* a device allocation failed                    */
  HSL_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed          */
  HSL_ERR_NAN_INPUT = 6,   /* W held a NaN (device-detected, via hsl_check) */
  HSL_ERR_TIMEOUT = 7      /* a bounded device wait gave up (via hsl_check) */
} hsl_status;

typedef enum { HSL_FMT_CSR = 0, HSL_FMT_NM24 = 1 } hsl_format;
typedef enum { HSL_F32 = 0, HSL_BF16 = 1 } hsl_dtype;

/* Create a layer handle for an m×n matrix with rank-r factors.
 *   fmt:   HSL_FMT_CSR (unstructured top-k S) or HSL_FMT_NM24 (2:4 S;
 *          needs n % 4 == 0).
 *   dtype: storage and arithmetic type of S values, U, V, X and Y
 *          (HSL_F32 or HSL_BF16); products accumulate in fp32.
 * Limits: 1 ≤ m, n; m·n < 2^31; 0 ≤ r ≤ 256.
 * Allocates nothing on the device; *out owns what later calls allocate.
 * [HSS] §Two-stage compression (the (S, U, V) triple), §Implementation. */
hsl_status hsl_create(int64_t m, int64_t n, int32_t r, hsl_format fmt,
                      hsl_dtype dtype, hsl_handle* out);

/* Release the handle and all device memory it owns.  Waits for the device
 * (cudaDeviceSynchronize on the handle's device) before freeing.  NULL is
 * a no-op.  The handle is the layer object of [HSS] §Implementation and
 * operational patterns, which holds (S, U, V) in place of the dense weight;
 * this ends its life. */
hsl_status hsl_destroy(hsl_handle h);

/* Stage 1: split W into S (kept in the handle) and the residual.
 *   W:        device, m×n row-major, element type w_dtype.
 *   frac:     CSR handles keep k = floor(frac·m·n) entries (frac ≤ 0 → 0,
 *             frac ≥ 1 → m·n), chosen by |w| descending with ties to the
 *             lower linear index i·n + j (exact radix select on the
 *             magnitude bits).  NM24 handles need frac == 0.5 and keep,
 *             in every group of 4 consecutive inputs of a row, the 2
 *             largest |w| (ties to the lower in-group index).
 *   residual: device, m×n of w_dtype, or NULL; receives W with the kept
 *             positions set to +0.0, bit-exact elsewhere.
 * S values are stored in the handle dtype (f32 → bf16 rounds to nearest
 * even; bf16 → f32 is exact).  A NaN in W is reported by hsl_check as
 * HSL_ERR_NAN_INPUT (the outputs are then meaningless but in bounds).
 * Invalidates any earlier hsl_pack.
 * [HSS] §Two-stage compression, Stage 1; [HASSLE] §3 for 2:4. */
hsl_status hsl_split_topk(hsl_handle h, const void* W, hsl_dtype w_dtype,
                          double frac, void* residual, hsl_stream s);

/* Top-k split that allocates no device memory.  The source pages have no
 * counterpart of this entry point: it exists for callers that may not call
 * cudaMalloc — code inside a serving runtime or plugin host that owns all
 * device memory and hands out pre-planned buffers, code that must not risk the
 * device-wide synchronisation of cudaMalloc/cudaFree, or callers without a
 * handle to keep workspace alive.  It computes exactly what hsl_split_topk
 * computes on a CSR handle (same kernels, bit-identical results), with every
 * input and output owned by the caller and no handle:
 *   W:        device, m×n row-major, element type w_dtype.
 *   frac:     k = floor(frac·m·n) kept (frac ≤ 0 → 0, frac ≥ 1 → m·n).
 *   row_ptr:  device int32[m+1];  col: device int32[k];  val: device, k values
 *             of val_dtype (f32 → bf16 rounds to nearest even).  col/val may
 *             be NULL when k == 0.
 *   residual: device m×n of w_dtype, or NULL.
 *   status:   device uint32, required (NULL → HSL_ERR_INVALID_ARG): it is the
 *             only channel for device-detected errors.  Cleared, then OR-ed
 *             with 1 for a NaN in W and 2 for a device wait that gave up.
 * Scratch: one fixed static device array of about 2.2 MB per GPU (held until
 * the process exits).  Limits: m ≤ 65536, n ≤ 2^31 − 1 and m·n < 2^31, else
 * HSL_ERR_UNSUPPORTED.  The first call on a device looks the array up with
 * that device current (make it before any stream capture).  All calls share
 * the array, so calls that can overlap on the GPU race: serialise them on one
 * stream.  Asynchronous on s, like the other entry points.
 * What it computes: [HSS] §Two-stage compression, Stage 1 (as hsl_split_topk). */
hsl_status hsl_split_topk_noalloc(const void* W, int64_t m, int64_t n, hsl_dtype w_dtype,
                                  double frac, int32_t* row_ptr, int32_t* col, void* val,
                                  hsl_dtype val_dtype, void* residual, uint32_t* status,
                                  hsl_stream s);

/* Number of stored sparse values (k for CSR, m·n/2 for NM24; 0 before any
 * split/set).  Host-only, no synchronisation (k is known on the host).
 * [HSS] §Two-stage compression, worked example: the count of kept weights
 * (52,428 for 5 % of a 1024×1024 matrix) that enters the parameter total. */
hsl_status hsl_get_nnz(hsl_handle h, int64_t* nnz);

/* Export the canonical S (stream-ordered device→device copies).
 * [HSS] §Two-stage compression, Stage 1: the kept weights are stored as a
 * sparse matrix in COO/CSR form; [HASSLE] §3 for the N:M form.
 *   CSR:  row_ptr[m+1] int32, col[nnz] int32 (ascending in each row),
 *         val[nnz] of the handle dtype; nm_idx unused (may be NULL).
 *   NM24: val[m][n/2] (the two kept values of each group, ascending column),
 *         nm_idx[m][n/4] uint8 = i0 | i1 << 2 with in-group indices
 *         i0 < i1; row_ptr/col unused (may be NULL). */
hsl_status hsl_get_sparse(hsl_handle h, int32_t* row_ptr, int32_t* col,
                          void* val, uint8_t* nm_idx, hsl_stream s);

/* Import a canonical CSR S (same layout as hsl_get_sparse), e.g. from a
 * checkpoint ([HSS] §Two-stage compression, Stage 1: S in COO/CSR form).  Columns must be < n; the handle trusts row_ptr to be
 * monotone with row_ptr[0] = 0 and row_ptr[m] = nnz.  CSR handles only.
 * Invalidates any earlier hsl_pack. */
hsl_status hsl_set_sparse_csr(hsl_handle h, int64_t nnz, const int32_t* row_ptr,
                              const int32_t* col, const void* val, hsl_stream s);

/* Import a canonical 2:4 S (layout as hsl_get_sparse; [HASSLE] §3, N:M
 * structured sparsity).  NM24 handles only.
 * Invalidates any earlier hsl_pack. */
hsl_status hsl_set_sparse_nm24(hsl_handle h, const void* val, const uint8_t* nm_idx,
                               hsl_stream s);

/* Build the device layouts hsl_apply streams: S repacked (CSR: rows padded
 * to 8 values with 16-bit column indices, [HSS] §Implementation (mixed
 * precision: narrow indices; the width is chosen by hsl_set_index_bits);
 * NM24: metadata interleaved per warp lane),
 * and copies of U [m][r] and V [n][r] (row-major, handle dtype, device).
 * Needs S (split or set) first, else HSL_ERR_NOT_READY. */
hsl_status hsl_pack(hsl_handle h, const void* U, const void* V, hsl_stream s);

/* Column-index width of the packed CSR S, used from the next hsl_pack on:
 *   16 — 16-bit columns (needs n < 65535); the default when n < 65535;
 *   32 — 32-bit columns (any n); the default when n ≥ 65535;
 *    8 — one delta byte per entry (column minus the previous entry's) plus a
 *        16-bit column base per 8-entry vector: 1.25 bytes per entry against
 *        2, so 3.25 instead of 4 streamed bytes per bf16 entry at decode.
 *        A gap of more than 255 columns inside a row takes filler entries
 *        (value 0, one per 255 columns); needs n < 65535 and each row's
 *        columns in ascending order (else hsl_pack returns HSL_ERR_UNSUPPORTED);
 *    0 — back to the default.
 * Large batches on the tensor cores use 16-bit columns; with another width
 * they run on the decode kernel.  CSR handles only; invalidates hsl_pack.
 * [HSS] §Implementation and operational patterns (from theory to production),
 * mixed precision: sparse indices as INT32 or in narrower integers (INT16,
 * INT8) to cut the memory of S further. */
hsl_status hsl_set_index_bits(hsl_handle h, int32_t bits);

/* Y = X Ŵᵀ, i.e. y = S x + U (Vᵀ x) for each of the batch rows of X.
 *   X: [batch][n], Y: [batch][m], handle dtype, row-major.  X and Y may be
 *   device pointers, or host pointers (pinned or pageable), in which case
 *   the call stages them through handle-owned device buffers with
 *   cudaMemcpyAsync on s (pinned Y: synchronise s before reading it).
 *   batch = 0 is a no-op.  Needs hsl_pack first, else HSL_ERR_NOT_READY.
 * [HSS] §Implementation and operational patterns, the forward
 * decomposition; [SQZ] §1 for why decode batches stream the weights. */
hsl_status hsl_apply(hsl_handle h, const void* X, void* Y, int64_t batch, hsl_stream s);

/* A group applies `count` independent layers in one pass (e.g. every
 * projection of a model at decode): one launch per kernel stage covers all of
 * them, with the rows of all layers split into CTA ranges of equal streamed
 * bytes.  All members must be packed and share format, dtype and device.
 * The group refers to the members' packed buffers: re-splitting, re-setting,
 * re-packing or destroying a member invalidates it (hsl_group_apply then
 * returns HSL_ERR_NOT_READY for a re-split member; create the group again).
 * Creating a group uploads its plan on s and synchronises s once.
 * [HSS] §Implementation and operational patterns (operating patterns): layers
 * are compressed and deployed one by one across a model's attention and MLP
 * projections; a group applies such a set of layers together. */
typedef struct hsl_group_s* hsl_group;
hsl_status hsl_group_create(const hsl_handle* hs, int32_t count, hsl_group* out, hsl_stream s);

/* Y[i] = apply(member i, X[i]) for every member; X[i] is [batch][n_i] and
 * Y[i] is [batch][m_i], device pointers.  The pointer tables are host
 * arrays; they are uploaded to the device only when they change.
 * Each member's product is the forward decomposition of hsl_apply ([HSS]
 * §Implementation and operational patterns; [SQZ] §1). */
hsl_status hsl_group_apply(hsl_group g, const void* const* X, void* const* Y, int64_t batch,
                           hsl_stream s);

/* Release the group (synchronises its device first).  NULL is a no-op.
 * [HSS] §Implementation and operational patterns (the layers held for the
 * forward pass), as hsl_group_create. */
hsl_status hsl_group_destroy(hsl_group g);

/* Stage 2 on the GPU: the rank-r factors of the residual R (device, m×n of
 * r_dtype; e.g. the residual hsl_split_topk wrote) as its truncated SVD with
 * √σ on each side, R ≈ U Vᵀ, U = U_r √Σ_r, V = V_r √Σ_r, computed by the
 * randomized range finder (Halko–Martinsson–Tropp) with the caller's Gaussian
 * test matrix:
 *   omega:       device fp32 [n][k], r ≤ k ≤ min(m, n, 512) (k − r is the
 *                oversampling);
 *   power_iters: q ≥ 0 subspace iterations (Y ← R Rᵀ Q, then Q = orth(Y));
 *   U [m][r], V [n][r]: device, handle dtype (pass them to hsl_pack);
 *   sigma [r]: device fp32, σ_1 ≥ … ≥ σ_r (0 where R has no such direction).
 * The tall products run on the tensor cores with fp32 operands split into
 * three bf16 terms (fp32-accurate); orthonormalisation and the small SVD use
 * fp64 Gram matrices and a Jacobi eigensolver.  Uses the handle's m, n, r and
 * dtype; allocates its workspace for the call (about 2·m·n·2 bytes for bf16
 * R) and synchronises s before freeing it.  r = 0 is a no-op.
 * [HSS] §Two-stage compression, Stage 2 (the residual factored into two
 * m×r / n×r matrices), and the implementation flow (low-rank factorisation,
 * O(n³)). */
hsl_status hsl_factor(hsl_handle h, const void* R, hsl_dtype r_dtype, const float* omega, int32_t k,
                      int32_t power_iters, void* U, void* V, float* sigma, hsl_stream s);

/* ---- Permutation for concentration ------------------------------------------
 * [HSS] §Permutation and hierarchical alignment: reorder the rows and columns
 * of W (reverse Cuthill–McKee) so that its large entries gather near the
 * diagonal, measure the gain with the concentration ratio
 *   ρ = Σ_{diagonal blocks} |W_ij| / Σ |W_ij|,
 * and keep the order so the layer is applied in the original order. */

/* ρ of W (device, m×n row-major, dtype): the diagonal blocks are the top-left
 * and bottom-right blocks of the 2×2 partition split at row ⌊m/2⌋ and column
 * ⌊n/2⌋; an all-zero W gives 0, a NaN in W gives NaN.  Sums in fp64 in a fixed
 * order (deterministic).  Writes *rho (host) and synchronises s.  Allocates a
 * small workspace for the call and frees it.
 * [HSS] §Permutation and hierarchical alignment (the ρ equation). */
hsl_status hsl_concentration(const void* W, int64_t m, int64_t n, hsl_dtype dtype, double* rho,
                             hsl_stream s);

/* Reverse Cuthill–McKee order of an m×n sparse pattern given as a HOST CSR
 * (row_ptr[m+1] from 0, col[row_ptr[m]] in [0, n)).  The graph is the
 * bipartite row–column graph (an edge per stored entry); start each component
 * at the unvisited vertex of least degree (ties: rows before columns, lower
 * index first), visit breadth first taking neighbours by increasing degree
 * (same ties), reverse the whole order.  row_order[k] / col_order[k] (host,
 * m and n int32) receive the original row / column placed k-th.  Runs on the
 * host (a one-off graph step); HSL_ERR_INVALID_ARG for a bad pattern.
 * [HSS] §Permutation and hierarchical alignment (reverse Cuthill–McKee). */
hsl_status hsl_rcm_order(int64_t m, int64_t n, const int32_t* row_ptr, const int32_t* col,
                         int32_t* row_order, int32_t* col_order);

/* out[k][l] = W[row_order[k]][col_order[l]] (device arrays; bit copies).  The
 * orders are copied to the host and checked to be permutations first
 * (HSL_ERR_INVALID_ARG otherwise), which synchronises s.
 * [HSS] §Permutation and hierarchical alignment (W permuted before the split). */
hsl_status hsl_permute(const void* W, int64_t m, int64_t n, hsl_dtype dtype,
                       const int32_t* row_order, const int32_t* col_order, void* out,
                       hsl_stream s);

/* Declare that the handle holds the permuted layer W' = W[row_order][:, col_order]
 * (split, set and packed from W'), so that hsl_apply returns the original
 * layer's output: x' = x[col_order], y' = Ŵ' x', y[row_order[k]] = y'[k].
 * Device arrays, copied into the handle after a host-side permutation check
 * (synchronises s).  NULL for both clears it.  Groups do not take permuted
 * layers.  [HSS] §Permutation and hierarchical alignment (outputs in the
 * original order). */
hsl_status hsl_set_permutation(hsl_handle h, const int32_t* row_order, const int32_t* col_order,
                               hsl_stream s);

/* Synchronise s and return, then clear, the device-side error of the handle
 * (HSL_ERR_NAN_INPUT, HSL_ERR_TIMEOUT) — HSL_OK if none.
 * [HSS] §Risks and mitigations, risk 1: keep the uncompressed weights as a
 * fallback for a compressed layer that misbehaves; this call is the detection
 * half of that, as a status. */
hsl_status hsl_check(hsl_handle h, hsl_stream s);

/* Static text for a status code (the statuses of hsl_check and of the
 * host-side checks; [HSS] §Risks and mitigations, risk 1, the same
 * detection-and-fallback passage). */
const char* hsl_status_str(hsl_status st);

/* Detail of the last failing call on this thread ("" if none).
 * [HSS] §Risks and mitigations, risk 1 (detection of a misbehaving layer),
 * as hsl_status_str. */
const char* hsl_last_message(void);

/* Number of kernels libhsl has launched in this process (all devices).
 * [HSS] §Implementation and operational patterns (actionable suggestions):
 * profile the compressed layers on the target hardware; this count lets a
 * profile tell the library's own kernels from everything else. */
uint64_t hsl_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* HSL_H_ */
