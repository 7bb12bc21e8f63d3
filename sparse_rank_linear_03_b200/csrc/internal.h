// Host-side internals of libhsl: the handle, device buffers, kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string>

#include "hsl.h"

namespace hsl {

// ---- bookkeeping -----------------------------------------------------------
extern std::atomic<uint64_t> g_launches;
inline void note_launch(int n = 1) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }
void set_message(const std::string& s);
hsl_status cuda_fail(cudaError_t e, const char* what);
// HSL_FAULT_INJECT=<what> (read on every call): host-side failure testing.
bool fault_injected(const char* what);

// cudaFuncSetAttribute(func, MaxDynamicSharedMemorySize, bytes) on the current
// device unless an earlier call already allowed at least `bytes` (grow-only), so
// a launch path makes the driver call once per kernel rather than per call.
cudaError_t allow_dyn_smem(const void* func, int bytes);
// cudaFuncSetAttribute(func, PreferredSharedMemoryCarveout, percent), once per
// device and function.
cudaError_t prefer_carveout(const void* func, int percent);

// Grow-only device allocation.
struct DevBuf {
  void* p = nullptr;
  size_t bytes = 0;
};
hsl_status ensure(DevBuf& b, size_t bytes, const char* what);
void release(DevBuf& b);

inline int dtype_bytes(hsl_dtype d) { return d == HSL_F32 ? 4 : 2; }
inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// ---- the apply problem descriptor (device-resident, one per layer) --------
struct ApplyProblem {
  const int32_t* prow;    // CSR: packed row starts (elements, multiples of 8), m+1
  const void* pcol;       // CSR: packed columns (pad = n): u16, u32, or u8 deltas
  const uint16_t* pbase;  // CSR, 8-bit columns: column of each 8-entry vector's first entry
  int32_t idx_bits;       // CSR: 8, 16 or 32
  const void* pval;       // CSR: packed values; NM24: values [m][n/2]
  const uint16_t* pmeta;  // NM24: metadata, interleaved per lane (see pack.cu)
  const void* U;          // [m][r_pad]
  const void* Vt;         // [r16][n]: V transposed, zero rows past r
  float* z;               // [16][r_pad]: z = Vᵀx per token of the batch chunk
  int32_t m, n, r_pad;
  int32_t group;          // CSR: lanes per row (4..32)
  int32_t meta_stride;    // NM24: u16 metadata words per row
  int32_t z_item0;        // this layer's first z work item (one per row of Vt)
  int32_t z_piece0;       // first (row, column piece) of Vt of this layer (in-kernel z)
  int64_t row0;           // first row of this layer in the concatenated row space
};

// Width of the pieces of a row of Vt that the in-kernel z sums (one warp
// each, at most 8 vectors of 8 per lane): ≥ 1024 columns, at most 16 pieces.
__host__ __device__ inline int z_piece_width(int n) {
  const int w = ((n + 15) / 16 + 255) / 256 * 256;
  return w < 1024 ? 1024 : w;
}

// Launch plan for one or more layers applied together.
struct ApplyPlan {
  int count = 0;
  hsl_format fmt = HSL_FMT_CSR;
  hsl_dtype dtype = HSL_F32;
  int32_t n_max = 0, r_pad_max = 0;
  int64_t rows_total = 0;
  int z_items = 0;      // z work items over all layers (0 when r == 0)
  int z_pieces = 0;     // (row, column piece) items of Vt over all layers
  int slices = 0;       // equal-byte row ranges the apply grid divides among CTAs
  bool vec16 = false;   // every layer has n % 16 == 0 (16-byte aligned 2:4 rows)
  int32_t idx_bits = 16;  // CSR column width of every member
  uint32_t* err = nullptr;  // error word the apply kernels report to (first member's)
  DevBuf probs;         // ApplyProblem[count]
  DevBuf prob_row0;     // int64[count+1]
  DevBuf cta_rows;      // int64[apply_grid+1]
  DevBuf xy_ptrs;       // const void*[2*count] (group calls)
  DevBuf zsync;         // two u64 counters: CTAs done with z, CTAs done with the call
  const void* const* last_x = nullptr;  // host cache of the uploaded pointers
  std::string host_xy;  // bytes of the last uploaded pointer table
};

struct Handle {
  int64_t m = 0, n = 0;
  int32_t r = 0, r_pad = 0;
  hsl_format fmt = HSL_FMT_CSR;
  hsl_dtype dtype = HSL_F32;
  int device = 0;
  int num_sms = 148;

  // canonical S
  DevBuf row_ptr, col, val;   // CSR
  DevBuf nm_val, nm_idx;      // NM24
  int64_t nnz = 0;
  bool has_sparse = false;

  // packed layouts
  DevBuf prow, pcol, pval, pmeta, pmeta_tc, U, Vt;
  int32_t group = 8, meta_stride = 0;
  bool csr_ascending = false;  // every packed row has strictly ascending columns
  int32_t index_bits = 0;       // requested column width (0: 16, or 32 when n ≥ 65535)
  int32_t idx_bits = 16;        // column width of the current pack
  DevBuf pbase, d8_lens;        // 8-bit columns: vector bases, row lengths with fillers
  int64_t pack_cap = 0;
  bool packed = false;

  // workspace
  DevBuf z, err, split_ws, flags;
  DevBuf tiles;  // per-tile counts of the sampled-bracket split
  DevBuf xstage, ystage, zpre;
  DevBuf sk_part, sk_cnt, sk_z;  // split-K small-batch apply: partial tiles, tile counters, z
  size_t sk_zcnt_off = 0, sk_zout_off = 0, sk_zpart_off = 0;  // in sk_z: counters, z, z pieces
  // permuted apply: the layer holds W' = W[row_order][:, col_order]
  DevBuf perm_row, perm_col, xperm, yperm;
  bool permuted = false;
  ApplyPlan plan;  // the single-layer plan, built by hsl_pack
};

// ---- launchers (each returns HSL_OK or an error already described) ------
hsl_status split_topk_run(Handle& h, const void* W, hsl_dtype wdt, int64_t k, void* R,
                          cudaStream_t s);
hsl_status split_24_run(Handle& h, const void* W, hsl_dtype wdt, void* R, cudaStream_t s);
hsl_status pack_sparse_run(Handle& h, cudaStream_t s);
hsl_status pack_factors_run(Handle& h, const void* U, const void* V, cudaStream_t s);
hsl_status csr_convert_run(Handle& h, const int32_t* row_ptr, const int32_t* col,
                           const void* val, cudaStream_t s);
hsl_status plan_build(ApplyPlan& plan, Handle* const* hs, int count, cudaStream_t s);
hsl_status apply_decode_run(ApplyPlan& plan, const void* X, void* Y, const void* const* xy_dev,
                            int64_t batch, int num_sms, cudaStream_t s);
// tensor-core path for large batches (2:4, bf16, n % 64 == 0)
constexpr int64_t kPrefillMinBatch = 65;
bool prefill_supported(const Handle& h, const void* X);
hsl_status apply_prefill_run(Handle& h, const void* X, void* Y, int64_t T, cudaStream_t s);
hsl_status prefill_z_run(Handle& h, const void* X, int64_t T, cudaStream_t s);
// CSR layers at large batches: each 64-column block of S densified into shared
// memory for dense tcgen05 MMAs (apply_prefill_csr.cu)
bool prefill_csr_supported(const Handle& h, const void* X);
hsl_status apply_prefill_csr_run(Handle& h, const void* X, void* Y, int64_t T, cudaStream_t s);
// small batches (2..64 tokens) of the same layers: sparse tensor cores with K
// split across every SM (apply_splitk.cu)
constexpr int64_t kSplitKMinBatch = 2, kSplitKMaxBatch = 64;
bool splitk_supported(const Handle& h, const void* X, int64_t T);
hsl_status apply_splitk_run(Handle& h, const void* X, void* Y, int64_t T, cudaStream_t s);
// Stage 2: randomized truncated SVD of the residual (factor.cu)
hsl_status factor_randomized_run(const void* R, int64_t m, int64_t n, hsl_dtype dtype, int r, int k,
                                 const float* omega, int power_iters, void* U, void* V,
                                 hsl_dtype out_dtype, float* sigma, uint32_t* err, int num_sms,
                                 cudaStream_t s);
// permutation for concentration (permute.cu)
hsl_status concentration_run(const void* W, int64_t m, int64_t n, hsl_dtype dt, double* out_dev,
                             double* partial, int blocks, cudaStream_t s);
int concentration_blocks(int64_t m);
hsl_status permute_run(const void* W, int64_t m, int64_t n, hsl_dtype dt, const int32_t* row_order,
                       const int32_t* col_order, void* out, cudaStream_t s);
hsl_status gather_cols_run(const void* x, int64_t batch, int64_t n, hsl_dtype dt,
                           const int32_t* order, void* out, cudaStream_t s);
hsl_status scatter_rows_run(const void* yp, int64_t batch, int64_t m, hsl_dtype dt,
                            const int32_t* order, void* y, cudaStream_t s);
hsl_status rcm_order(int64_t m, int64_t n, const int32_t* row_ptr, const int32_t* col,
                     int32_t* row_order, int32_t* col_order);
// 2-D row-major TMA map: rows × cols elements, box {box_cols, box_rows}
// (apply_prefill.cu); false when the driver entry point or the encoding fails.
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base,
                  int64_t rows, int64_t cols, int64_t row_stride_elems, int box_cols,
                  int box_rows, CUtensorMapSwizzle sw);
// 3-D TMA map over a row-major bf16 [rows][cols] matrix (cols a multiple of 64)
// seen as [cols / 64][rows][64]: a box {64, box_rows, box_kblocks} brings
// box_kblocks 64-column K-blocks of box_rows rows, each K-block's rows
// contiguous (128-byte swizzle), in one copy (apply_prefill.cu).
bool make_tmap_kblocks(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                       int box_rows, int box_kblocks);
bool tmap_available();

}  // namespace hsl

struct hsl_handle_s {
  hsl::Handle h;
};
