// Stage 1, unstructured: exact magnitude top-k split of W into CSR S + residual.
//
// "Hierarchical Sparse + Low-Rank Compression of LLMs", §Two-stage
// hierarchical sparse + low-rank compression, Stage 1: the largest-|w|
// fraction of the weights goes into a sparse (COO/CSR) matrix, the rest is the
// dense residual.  k = floor(frac·m·n) entries are kept over the whole matrix;
// ties in |w| go to the lower linear index i·n + j.
//
// Design (B200):
//   1. Radix select on the magnitude bits (sign cleared; order of the key
//      bits = order of |w| for every non-NaN value, ±0 equal, Inf largest).
//      bf16 keys have 15 bits: ONE streaming pass with a 32768-bin histogram
//      per CTA in shared memory (128 KB) finds the threshold key T exactly.
//      fp32 keys (31 bits) take three passes of 11/11/9 bits.
//   2. One emit pass over W, persistent CTAs taking blocks of rows (up to 32K
//      elements, held in registers) in ticket order.  Each block's counts of
//      keys > T and keys == T are published and the exclusive prefix over
//      earlier blocks comes from a decoupled look-back, 32 predecessors per
//      poll (bounded spin; CTAs only wait on blocks whose tickets were taken
//      earlier, so they are running).  An element's CSR position is
//      gt_before + min(need, eq_before), need = k − #(key > T): ties are taken
//      in linear order.  Per 16-byte vector the masks of keys > T / == T come
//      from one carry-free packed subtraction per threshold (bf16); the kept
//      elements are walked by their set bits; the residual is the vector with
//      those elements zeroed (bit copy, +0.0 where kept).  Rows wider than a
//      register block use a per-row variant of the same scheme.
//   HBM traffic: bf16 2 reads of W + 1 write of R + S; fp32 4 reads.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "split_kernels.cuh"

namespace hsl {
namespace {

template <typename KT, typename SB>
hsl_status emit_launch(Handle& h, const KT* W, int64_t k, KT* R, SelState* st, unsigned* ticket,
                       unsigned long long* flags, uint32_t* err, bool vec_ok, cudaStream_t s) {
  constexpr int EPV = 16 / sizeof(KT);
  const int64_t cap = int64_t(kEmitThreads) * kVPT * EPV;
  if (vec_ok && h.n <= cap) {
    const int rb = int(cap / h.n);
    const int64_t nblk = (h.m + rb - 1) / rb;
    static int occ_blk = 0;
    if (!occ_blk)
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_blk, k_split_emit_blk<KT, SB>,
                                                    kEmitThreads, 0);
    const int64_t grid = std::min<int64_t>(nblk, int64_t(h.num_sms) * std::max(occ_blk, 1));
    k_split_emit_blk<KT, SB><<<unsigned(grid), kEmitThreads, 0, s>>>(
        W, h.m, h.n, rb, nblk, st, ticket, flags, static_cast<int32_t*>(h.row_ptr.p),
        static_cast<int32_t*>(h.col.p), static_cast<SB*>(h.val.p), R, k,
        static_cast<uint32_t*>(h.err.p));
    note_launch();
    return cuda_fail(cudaGetLastError(), "split emit launch");
  }
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_split_emit<KT, SB>, kEmitThreads, 0);
  const int64_t grid = std::min<int64_t>(h.m, int64_t(h.num_sms) * std::max(occ, 1));
  k_split_emit<KT, SB><<<unsigned(grid), kEmitThreads, 0, s>>>(
      W, h.m, h.n, st, ticket, flags, static_cast<int32_t*>(h.row_ptr.p),
      static_cast<int32_t*>(h.col.p), static_cast<SB*>(h.val.p), R, k,
      static_cast<uint32_t*>(h.err.p), vec_ok ? 1 : 0);
  note_launch();
  return cuda_fail(cudaGetLastError(), "split emit launch");
}

template <typename KT>
hsl_status run_typed(Handle& h, const KT* W, int64_t k, KT* R, cudaStream_t s) {
  const int64_t count = h.m * h.n;
  // workspace: hist[32768] | SelState | ticket  ; flags[m] separately
  const size_t hist_bytes = 32768 * sizeof(unsigned);
  if (hsl_status e = ensure(h.split_ws, hist_bytes + 256, "split workspace")) return e;
  if (hsl_status e = ensure(h.flags, size_t(h.m) * 8, "split look-back flags")) return e;
  char* ws = static_cast<char*>(h.split_ws.p);
  unsigned* hist = reinterpret_cast<unsigned*>(ws);
  SelState* st = reinterpret_cast<SelState*>(ws + hist_bytes);
  unsigned* ticket = reinterpret_cast<unsigned*>(ws + hist_bytes + 64);
  unsigned long long* flags = static_cast<unsigned long long*>(h.flags.p);
  uint32_t* err = static_cast<uint32_t*>(h.err.p);

  const bool vec_ok = (reinterpret_cast<uintptr_t>(W) % 16 == 0) &&
                      (R == nullptr || reinterpret_cast<uintptr_t>(R) % 16 == 0) &&
                      ((h.n * int64_t(sizeof(KT))) % 16 == 0);

  if (k == 0) {
    // nothing is kept: T above every key, need = 0
    // (the one histogram pass below still scans W for NaN)
    k_sel_init<<<1, 1, 0, s>>>(st, 0u, 0xFFFFFFFFu);
    note_launch();
  } else {
    k_sel_init<<<1, 1, 0, s>>>(st, uint32_t(k), 0u);
    note_launch();
  }

  int passes, bits[3], shifts[3];
  if (sizeof(KT) == 2) {
    passes = 1; bits[0] = 15; shifts[0] = 0;
  } else {
    passes = 3; bits[0] = 11; shifts[0] = 20; bits[1] = 11; shifts[1] = 9; bits[2] = 9; shifts[2] = 0;
  }
  const int hist_grid = h.num_sms;
  for (int p = 0; p < passes; ++p) {
    if (k == 0 && p > 0) break;
    if (cudaError_t e = cudaMemsetAsync(hist, 0, hist_bytes, s)) return cuda_fail(e, "memset");
    const size_t smem = (size_t(1) << bits[p]) * sizeof(unsigned);
    if (bits[p] == 15) {
      auto kern = k_split_hist<KT, 15>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      kern<<<hist_grid, 1024, smem, s>>>(W, count, st, shifts[p], hist, err, vec_ok ? 1 : 0);
    } else if (bits[p] == 11) {
      k_split_hist<KT, 11><<<hist_grid * 2, 1024, smem, s>>>(W, count, st, shifts[p], hist, err,
                                                              vec_ok ? 1 : 0);
    } else {
      k_split_hist<KT, 9><<<hist_grid * 2, 1024, smem, s>>>(W, count, st, shifts[p], hist, err,
                                                             vec_ok ? 1 : 0);
    }
    note_launch();
    if (hsl_status e = cuda_fail(cudaGetLastError(), "split histogram launch")) return e;
    if (k > 0) {
      k_split_select<<<1, 1024, 0, s>>>(hist, 1 << bits[p], shifts[p], st);
      note_launch();
      if (hsl_status e = cuda_fail(cudaGetLastError(), "split select launch")) return e;
    }
  }

  if (cudaError_t e = cudaMemsetAsync(ticket, 0, 4, s)) return cuda_fail(e, "memset");
  if (cudaError_t e = cudaMemsetAsync(flags, 0, size_t(h.m) * 8, s)) return cuda_fail(e, "memset");
  if (h.dtype == HSL_BF16)
    return emit_launch<KT, uint16_t>(h, W, k, R, st, ticket, flags, err, vec_ok, s);
  return emit_launch<KT, uint32_t>(h, W, k, R, st, ticket, flags, err, vec_ok, s);
}

}  // namespace

hsl_status split_topk_run(Handle& h, const void* W, hsl_dtype wdt, int64_t k, void* R,
                          cudaStream_t s) {
  const size_t vb = size_t(dtype_bytes(h.dtype));
  if (hsl_status e = ensure(h.row_ptr, size_t(h.m + 1) * 4, "CSR row_ptr")) return e;
  if (hsl_status e = ensure(h.col, size_t(std::max<int64_t>(k, 1)) * 4, "CSR col")) return e;
  if (hsl_status e = ensure(h.val, size_t(std::max<int64_t>(k, 1)) * vb, "CSR val")) return e;
  if (wdt == HSL_BF16)
    return run_typed<uint16_t>(h, static_cast<const uint16_t*>(W), k, static_cast<uint16_t*>(R), s);
  return run_typed<uint32_t>(h, static_cast<const uint32_t*>(W), k, static_cast<uint32_t*>(R), s);
}

}  // namespace hsl
