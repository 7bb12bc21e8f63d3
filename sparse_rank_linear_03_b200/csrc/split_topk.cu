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
//      fp32 keys (31 bits) take three passes of 11/11/9 bits.  Large bf16
//      splits first bracket T from a 1/64 sample of W (runs of 256 elements
//      at hashed offsets); the pass then counts keys above the bracket with
//      packed compares and histograms only the keys inside it.  If T falls
//      outside, the full histogram pass runs (it and its select are launched
//      always and return at once when the bracket held T).
//   2. One emit pass over W (k_split_emit_tile).  Persistent CTAs take tiles
//      of W in ticket order and keep three in flight by 1-D bulk copies into
//      shared memory.  An element's CSR position is
//      gt_before + min(need, eq_before), need = k − #(key > T): ties are taken
//      in linear order.  A tile's (gt, eq) prefix over the tiles before it comes
//      from the per-tile counts that the bracket pass recorded (16 KB tiles,
//      four CTAs per SM), or else from a decoupled look-back (32 KB tiles,
//      32 predecessors per poll, bounded spin; CTAs only wait on tiles whose
//      tickets were taken earlier, so those tiles' CTAs are running).  Per
//      16-byte vector, the masks of keys > T and == T come from one carry-free
//      packed subtraction per threshold (bf16).  A tile's S entries are written
//      in output order with coalesced stores.  The kept elements are zeroed in
//      the staged tile, and a bulk store writes it back as the residual (a bit
//      copy, +0.0 where kept).  When W or R is not 16-byte aligned, a per-row
//      variant of the same scheme (k_split_emit) runs instead.
//   HBM traffic: bf16 2 reads of W + 1 write of R + S; fp32 4 reads.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "split_kernels.cuh"

namespace hsl {
namespace {

template <typename KT, typename SB, int TB>
hsl_status emit_tiles(Handle& h, const KT* W, int64_t k, KT* R, SelState* st, unsigned* ticket,
                      unsigned long long* flags, uint32_t* err, const Bracket* br,
                      const unsigned long long* tile_pre, cudaStream_t s) {
  constexpr int TE = TB / int(sizeof(KT));
  const int64_t count = h.m * h.n;
  const int64_t ntiles = (count + TE - 1) / TE;
  const size_t smem = size_t(kStages) * TB;
  auto kern = k_split_emit_tile<KT, SB, TB>;
  if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(kern), int(smem)))
    return cuda_fail(e, "split emit smem attribute");
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kTileThreads, smem);
  const int64_t grid = std::min<int64_t>(ntiles, int64_t(h.num_sms) * std::max(occ, 1));
  kern<<<unsigned(std::max<int64_t>(grid, 1)), kTileThreads, smem, s>>>(
      W, h.m, count, make_fastdiv(uint32_t(h.n)), ntiles, st, ticket, flags,
      static_cast<int32_t*>(h.row_ptr.p), static_cast<int32_t*>(h.col.p),
      static_cast<SB*>(h.val.p), R, k, err, br, tile_pre);
  note_launch();
  return cuda_fail(cudaGetLastError(), "split emit launch");
}

template <typename KT, typename SB>
hsl_status emit_launch(Handle& h, const KT* W, int64_t k, KT* R, SelState* st, unsigned* ticket,
                       unsigned long long* flags, uint32_t* err, bool vec_ok, const Bracket* br,
                       const unsigned long long* tile_pre, cudaStream_t s) {
  if (vec_ok) {
    // the tile size of the bracket pass's per-tile counts, else look-back tiles
    return tile_pre ? emit_tiles<KT, SB, kTileBytesPre>(h, W, k, R, st, ticket, flags, err, br,
                                                        tile_pre, s)
                    : emit_tiles<KT, SB, kTileBytesLB>(h, W, k, R, st, ticket, flags, err, br,
                                                       tile_pre, s);
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
  // workspace: hist[32768] | sample hist[32768] | SelState | ticket | Bracket ; flags separately
  const size_t hist_bytes = 32768 * sizeof(unsigned);
  if (hsl_status e = ensure(h.split_ws, 2 * hist_bytes + 256, "split workspace")) return e;
  // look-back flags: one per row (per-row emit) or per tile (at most one per
  // tile of the smaller size)
  const int64_t nflags = std::max<int64_t>(h.m, (count * int64_t(sizeof(KT)) + kTileBytesPre - 1) / kTileBytesPre);
  if (hsl_status e = ensure(h.flags, size_t(nflags) * 8, "split look-back flags")) return e;
  char* ws = static_cast<char*>(h.split_ws.p);
  unsigned* hist = reinterpret_cast<unsigned*>(ws);
  unsigned* shist = reinterpret_cast<unsigned*>(ws + hist_bytes);
  SelState* st = reinterpret_cast<SelState*>(ws + 2 * hist_bytes);
  unsigned* ticket = reinterpret_cast<unsigned*>(ws + 2 * hist_bytes + 64);
  Bracket* br = reinterpret_cast<Bracket*>(ws + 2 * hist_bytes + 128);
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
  const uint32_t* skip = nullptr;
  const Bracket* brk = nullptr;
  const unsigned long long* tile_pre = nullptr;
  const int64_t nstrata = count / 8 / kSampleStride;
  if (sizeof(KT) == 2 && vec_ok && k > 0 && count >= (int64_t(1) << 22) &&
      count < (int64_t(1) << 32)) {
    // sampled bracket: the full histogram pass below then runs only if the
    // threshold fell outside it
    const double S = double(nstrata) * kSampleRun * 8;
    const double ks = double(k) * S / double(count);
    const double margin = ks / 32 + 16 * std::sqrt(ks) + 4096;
    const uint32_t r_hi = uint32_t(std::max(0.0, std::floor(ks - margin)));
    const uint32_t r_lo = uint32_t(std::min(S + 1, std::ceil(ks + margin)));
    if (cudaError_t e = cudaMemsetAsync(hist, 0, 2 * hist_bytes, s)) return cuda_fail(e, "memset");
    const int smem = int(hist_bytes);
    if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_sample_hist), smem))
      return cuda_fail(e, "split sample smem attribute");
    if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_count_bracket), smem))
      return cuda_fail(e, "split count smem attribute");
    const uint16_t* W16 = reinterpret_cast<const uint16_t*>(W);
    // per emit tile: count above the bracket, bracket histogram, counts, prefixes
    const int64_t ntiles = (count * 2 + kTileBytesPre - 1) / kTileBytesPre;
    const size_t tb_above = size_t(ntiles) * 4, tb_hist = size_t(ntiles) * kTileBins * 4;
    if (hsl_status e = ensure(h.tiles, tb_above + tb_hist + size_t(ntiles) * 16 + 64, "split tiles"))
      return e;
    char* tb = static_cast<char*>(h.tiles.p);
    uint32_t* tile_above = reinterpret_cast<uint32_t*>(tb);
    uint32_t* tile_hist = reinterpret_cast<uint32_t*>(tb + tb_above);
    unsigned long long* tile_cnt =
        reinterpret_cast<unsigned long long*>(tb + round_up(int64_t(tb_above + tb_hist), 16));
    unsigned long long* pre = tile_cnt + ntiles;
    k_sample_hist<<<hist_grid, 1024, smem, s>>>(W16, nstrata, shist);
    k_bracket_select<<<1, 1024, 0, s>>>(shist, r_hi, r_lo, br);
    k_count_bracket<<<hist_grid, 1024, smem, s>>>(W16, count / 8, br, hist, err, tile_above,
                                                  tile_hist);
    k_bracket_finish<<<1, 1024, 0, s>>>(hist, br, st, uint32_t(k));
    k_tile_counts<<<hist_grid * 2, 256, 0, s>>>(tile_above, tile_hist, ntiles, br, st, tile_cnt);
    k_tile_scan<<<1, 1024, 0, s>>>(tile_cnt, ntiles, br, pre);
    note_launch(6);
    if (hsl_status e = cuda_fail(cudaGetLastError(), "split bracket launch")) return e;
    skip = &br->ok;
    brk = br;
    tile_pre = pre;
  }
  for (int p = 0; p < passes; ++p) {
    if (k == 0 && p > 0) break;
    if (!skip)  // after a bracket, hist is already zero wherever the full pass needs it
      if (cudaError_t e = cudaMemsetAsync(hist, 0, hist_bytes, s)) return cuda_fail(e, "memset");
    const size_t smem = (size_t(1) << bits[p]) * sizeof(unsigned);
    if (bits[p] == 15) {
      auto kern = k_split_hist<KT, 15>;
      if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(kern), int(smem)))
        return cuda_fail(e, "split histogram smem attribute");
      kern<<<hist_grid, 1024, smem, s>>>(W, count, st, shifts[p], hist, err, vec_ok ? 1 : 0, skip);
    } else if (bits[p] == 11) {
      k_split_hist<KT, 11><<<hist_grid * 2, 1024, smem, s>>>(W, count, st, shifts[p], hist, err,
                                                              vec_ok ? 1 : 0, skip);
    } else {
      k_split_hist<KT, 9><<<hist_grid * 2, 1024, smem, s>>>(W, count, st, shifts[p], hist, err,
                                                             vec_ok ? 1 : 0, skip);
    }
    note_launch();
    if (hsl_status e = cuda_fail(cudaGetLastError(), "split histogram launch")) return e;
    if (k > 0) {
      k_split_select<<<1, 1024, 0, s>>>(hist, 1 << bits[p], shifts[p], st, skip);
      note_launch();
      if (hsl_status e = cuda_fail(cudaGetLastError(), "split select launch")) return e;
    }
  }

  if (cudaError_t e = cudaMemsetAsync(ticket, 0, 4, s)) return cuda_fail(e, "memset");
  if (cudaError_t e = cudaMemsetAsync(flags, 0, size_t(nflags) * 8, s)) return cuda_fail(e, "memset");
  if (h.dtype == HSL_BF16)
    return emit_launch<KT, uint16_t>(h, W, k, R, st, ticket, flags, err, vec_ok, brk, tile_pre, s);
  return emit_launch<KT, uint32_t>(h, W, k, R, st, ticket, flags, err, vec_ok, brk, tile_pre, s);
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
