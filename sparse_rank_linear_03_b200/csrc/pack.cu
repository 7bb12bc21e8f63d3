// Packing: canonical S → the layouts the apply kernels stream, padded factor
// copies, and the launch plan (row ranges of equal streamed bytes per CTA).
//
// "Hierarchical Sparse + Low-Rank Compression of LLMs", §Implementation and
// operational patterns (from theory to production), mixed precision: the
// pages store factors in 16 bits and sparse indices in narrow integers.  The
// packed CSR uses 16-bit column indices (n < 65535) and pads each row to a
// multiple of 8 entries so every lane reads whole 16-byte vectors; padding
// entries point at column n, a zero kept at the end of the staged x.
//
// Packed 2:4 metadata: one 16-bit word per chunk of 8 kept values (4 groups,
// 4 bits each = i0 | i1 << 2).  Within a row, chunk q = (8·s + t)·32 + l is
// stored at word s·256 + l·8 + t, so lane l of a warp fetches the metadata of
// its next 8 chunks with a single 16-byte load.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace hsl {
namespace {

__device__ __forceinline__ int32_t pad8(int32_t v) { return (v + 7) & ~7; }

// One CTA: prow = exclusive scan of the padded row lengths; prow[m] = total.
// A row whose bounds are not 0 <= row_ptr[i] <= row_ptr[i+1] <= nnz is taken
// as empty and flagged; starts are clamped to cap so no later read or write
// leaves the packed arrays, whatever an imported row_ptr holds.
__device__ __forceinline__ int32_t row_len_checked(const int32_t* row_ptr, int64_t i, int64_t nnz,
                                                   bool& bad) {
  const int32_t a = row_ptr[i], b = row_ptr[i + 1];
  if (a < 0 || b < a || int64_t(b) > nnz) {
    bad = true;
    return 0;
  }
  return b - a;
}

// lens (optional): the row lengths to pad, in place of row_ptr's differences
// (the 8-bit layout adds filler entries to rows).
__global__ void __launch_bounds__(1024) k_csr_prow(const int32_t* __restrict__ row_ptr, int64_t m,
                                                   int64_t nnz, int64_t cap,
                                                   int32_t* __restrict__ prow, uint32_t* err,
                                                   const int32_t* __restrict__ lens) {
  __shared__ int64_t wsum[32];
  const int t = threadIdx.x, nt = blockDim.x;
  const int64_t per = (m + nt - 1) / nt;
  const int64_t lo = int64_t(t) * per < m ? int64_t(t) * per : m;
  const int64_t hi = lo + per < m ? lo + per : m;
  bool bad = false;
  int64_t s = 0;
  auto len_of = [&](int64_t i) {
    const int32_t l = row_len_checked(row_ptr, i, nnz, bad);
    return lens ? lens[i] : l;
  };
  for (int64_t i = lo; i < hi; ++i) s += pad8(len_of(i));
  int64_t incl = s;
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if ((t & 31) >= o) incl += v;
  }
  if ((t & 31) == 31) wsum[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    const int64_t w = t < (nt >> 5) ? wsum[t] : 0;
    int64_t wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, wi, o);
      if (t >= o) wi += v;
    }
    wsum[t] = wi - w;
  }
  __syncthreads();
  int64_t off = wsum[t >> 5] + incl - s;
  for (int64_t i = lo; i < hi; ++i) {
    prow[i] = int32_t(off < cap ? off : cap);
    off += pad8(len_of(i));
  }
  if (hi == m && lo < hi) {
    if (off > cap) bad = true;
    prow[m] = int32_t(off < cap ? off : cap);
  }
  if (m == 0 && t == 0) prow[0] = 0;
  if (t == 0 && row_ptr[0] != 0) bad = true;
  if (bad) set_error(err, kErrBadIndex);
}

// Warp per row: copy columns (int32 → the packed column type) and values;
// pad with (n, 0).  order_flag bit 0: a row's columns are not strictly
// ascending; bit 1: a row's columns decrease somewhere.
template <typename SB, typename CT>
__global__ void __launch_bounds__(256) k_csr_fill(const int32_t* __restrict__ row_ptr,
                                                  const int32_t* __restrict__ col,
                                                  const SB* __restrict__ val,
                                                  const int32_t* __restrict__ prow, int64_t m,
                                                  int64_t nnz, int32_t n, CT* __restrict__ pcol,
                                                  SB* __restrict__ pval, uint32_t* err,
                                                  uint32_t* order_flag) {
  const int lane = threadIdx.x & 31;
  bool bad = false, unordered = false, descending = false;
  for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; i < m;
       i += (int64_t(gridDim.x) * blockDim.x) >> 5) {
    bool badrow = false;
    const int32_t len = row_len_checked(row_ptr, i, nnz, badrow);
    const int32_t s0 = row_ptr[i];
    const int32_t d0 = prow[i], plen = prow[i + 1] - d0;
    for (int32_t e = lane; e < plen; e += 32) {
      bool in = e < len;
      const int32_t c = in ? col[s0 + e] : n;
      if (in && (c < 0 || c >= n)) {  // never index outside the staged x
        bad = true;
        in = false;
      }
      pcol[d0 + e] = in ? CT(c) : CT(n);
      pval[d0 + e] = in ? val[s0 + e] : SB(0);
      // the large-batch CSR path needs strictly ascending columns in a row
      if (in && e > 0 && c <= col[s0 + e - 1]) unordered = true;
      if (in && e > 0 && c < col[s0 + e - 1]) descending = true;
    }
  }
  if (bad) set_error(err, kErrBadIndex);
  if (unordered || descending) atomicOr(order_flag, (unordered ? 1u : 0u) | (descending ? 2u : 0u));
}

// 8-bit layout: a filler entry (value 0) goes before every entry whose column
// is more than 255 past the previous one, once per 255 columns of the gap.
__device__ __forceinline__ int32_t d8_fillers(int32_t gap) { return gap > 255 ? (gap - 1) / 255 : 0; }

// Thread per row: the row length in the 8-bit layout (entries + fillers).
// Rows whose columns decrease are flagged (order_flag bit 1) and counted as
// they are; the pack then refuses the layout.
__global__ void k_csr_d8_len(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                             int64_t m, int64_t nnz, int32_t n, int32_t* __restrict__ lens,
                             uint32_t* order_flag) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < m;
       i += int64_t(gridDim.x) * blockDim.x) {
    bool bad = false;
    const int32_t len = row_len_checked(row_ptr, i, nnz, bad);
    const int32_t s0 = bad ? 0 : row_ptr[i];
    int32_t extra = 0, prev = -1;
    bool first = true;
    for (int32_t e = 0; e < len; ++e) {
      const int32_t c = col[s0 + e];
      if (c < 0 || c >= n) continue;  // dropped by the fill as well
      if (!first) {
        if (c < prev) atomicOr(order_flag, 2u);
        else extra += d8_fillers(c - prev);
      }
      prev = c;
      first = false;
    }
    lens[i] = len + extra;
  }
}

// Thread per row: values, one delta byte per entry (column minus the previous
// entry's; 0 for the first entry of an 8-entry vector, whose column is the
// vector's 16-bit base), fillers (value 0, delta 255) and padding (value 0,
// delta 0) up to the padded length.
template <typename SB>
__global__ void k_csr_d8_fill(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                              const SB* __restrict__ val, const int32_t* __restrict__ prow,
                              int64_t m, int64_t nnz, int32_t n, uint8_t* __restrict__ pdelta,
                              uint16_t* __restrict__ pbase, SB* __restrict__ pval, uint32_t* err) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < m;
       i += int64_t(gridDim.x) * blockDim.x) {
    bool bad = false;
    const int32_t len = row_len_checked(row_ptr, i, nnz, bad);
    const int32_t s0 = bad ? 0 : row_ptr[i];
    const int32_t d0 = prow[i], d1 = prow[i + 1];
    int32_t pos = d0, prev = 0;
    auto put = [&](int32_t c, SB v) {
      if (pos >= d1) return;  // never past the row's packed slots
      const bool vstart = ((pos - d0) & 7) == 0;
      pdelta[pos] = vstart ? uint8_t(0) : uint8_t(c - prev);
      if (vstart) pbase[pos >> 3] = uint16_t(c);
      pval[pos] = v;
      prev = c;
      ++pos;
    };
    bool first = true, badcol = false;
    for (int32_t e = 0; e < len; ++e) {
      const int32_t c = col[s0 + e];
      if (c < 0 || c >= n) {
        badcol = true;
        continue;
      }
      if (!first && c >= prev)
        for (int32_t f = d8_fillers(c - prev); f > 0; --f) put(prev + 255, SB(0));
      put(c, val[s0 + e]);
      first = false;
    }
    const int32_t last = first ? 0 : prev;
    while (pos < d1) put(last, SB(0));
    if (badcol) set_error(err, kErrBadIndex);
  }
}

__global__ void k_nm24_meta(const uint8_t* __restrict__ idx, int64_t m, int64_t n,
                            int32_t meta_stride, uint16_t* __restrict__ pmeta) {
  const int64_t words = m * meta_stride;
  const int64_t groups = n / 4;
  for (int64_t w = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; w < words;
       w += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = w / meta_stride;
    const int32_t pos = int32_t(w % meta_stride);
    const int32_t s = pos >> 8, l = (pos & 255) >> 3, t = pos & 7;
    const int64_t q = int64_t(s * 8 + t) * 32 + l;
    uint32_t word = 0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int64_t grp = 4 * q + g;
      if (grp < groups) word |= uint32_t(idx[row * groups + grp] & 0xF) << (4 * g);
    }
    pmeta[w] = uint16_t(word);
  }
}

template <typename SB>
__global__ void k_pad_cols(const SB* __restrict__ src, int64_t rows, int32_t r, int32_t r_pad,
                           SB* __restrict__ dst) {
  const int64_t total = rows * r_pad;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = e / r_pad;
    const int32_t c = int32_t(e % r_pad);
    dst[e] = c < r ? src[i * r + c] : SB(0);
  }
}

// Vt[c][j] = V[j][c] for c < r, zero rows up to r16: V as given ([n][r],
// row-major) transposed through 32×32 shared-memory tiles so both sides are
// coalesced.  The decode z = Vᵀx reads whole rows of Vt, the prefill Z = X·V
// takes it as its B operand.
template <typename SB>
__global__ void k_transpose_pad(const SB* __restrict__ V, int64_t n, int32_t r, int32_t r16,
                                SB* __restrict__ Vt) {
  __shared__ SB tile[32][33];
  const int64_t tiles_j = (n + 31) / 32, tiles_c = (r16 + 31) / 32;
  for (int64_t tt = blockIdx.x; tt < tiles_j * tiles_c; tt += gridDim.x) {
    const int64_t j0 = (tt % tiles_j) * 32;
    const int32_t c0 = int32_t(tt / tiles_j) * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {  // rows j of V, columns c
      const int64_t j = j0 + i;
      const int32_t c = c0 + int32_t(threadIdx.x);
      tile[i][threadIdx.x] = (j < n && c < r) ? V[j * r + c] : SB(0);
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {  // rows c of Vt, columns j
      const int32_t c = c0 + i;
      const int64_t j = j0 + threadIdx.x;
      if (c < r16 && j < n) Vt[int64_t(c) * n + j] = tile[threadIdx.x][i];
    }
    __syncthreads();
  }
}

// 2:4 metadata for the sparse tensor-core prefill: one uint2 per (128-row
// tile, 64-column K-block, TMEM lane L).  Word i feeds the sparse MMA over
// logical columns [64·kb + 32·i, +32).  Lane L = 16·m2 + 8·k1 + m0 holds in its
// low / high 16 bits the four nibbles (16 columns, half k1) of tile rows
// m0 + 16·m2 and m0 + 8 + 16·m2 — rows i and i + 8 share a word, the pairing
// of the warp-level sparse MMAs.  Rows past m get the valid pattern 0x4
// (their values are zero).
__device__ __forceinline__ uint32_t nib4(const uint8_t* idx, int64_t groups, int64_t row, int64_t g0,
                                         int64_t m) {
  if (row >= m) return 0x4444u;
  const uint8_t* p = idx + row * groups + g0;
  return uint32_t(p[0] & 0xF) | (uint32_t(p[1] & 0xF) << 4) | (uint32_t(p[2] & 0xF) << 8) |
         (uint32_t(p[3] & 0xF) << 12);
}

__global__ void k_meta_tc(const uint8_t* __restrict__ idx, int64_t m, int64_t n,
                          uint2* __restrict__ out) {
  const int64_t nkb = n / 64, groups = n / 4;
  const int64_t total = ((m + 127) / 128) * nkb * 128;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int L = int(e % 128);
    const int64_t kb = (e / 128) % nkb, mt = e / (128 * nkb);
    const int m0 = L & 7, k1 = (L >> 3) & 1, m2 = L >> 4;
    const int64_t rlo = mt * 128 + m0 + 16 * m2, rhi = rlo + 8;
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int64_t g0 = 16 * kb + 8 * i + 4 * k1;
      w[i] = nib4(idx, groups, rlo, g0, m) | (nib4(idx, groups, rhi, g0, m) << 16);
    }
    out[e] = make_uint2(w[0], w[1]);
  }
}

// One CTA: boundaries of `slices` row ranges of equal streamed bytes over the
// concatenated rows of all layers.  Cost of the first i rows of layer p:
//   CSR : prow[i]·(value + 2 index bytes) + i·(U row bytes + 8)
//   NM24: i·(n/2 value bytes + n/8 metadata bytes + U row bytes + 8)
__global__ void __launch_bounds__(1024) k_partition(const ApplyProblem* __restrict__ probs,
                                                    int count, int fmt_csr, int eb,
                                                    int64_t* __restrict__ cost0, int slices,
                                                    int64_t* __restrict__ cta_rows) {
  auto row_cost = [&](const ApplyProblem& P, int64_t i) -> int64_t {
    const int64_t u = int64_t(P.r_pad) * eb + 8;
    // per packed entry, in quarter bytes: the value and its column (8-bit
    // deltas carry a 16-bit base per 8 entries)
    const int64_t q = 4 * eb + (P.idx_bits == 8 ? 5 : P.idx_bits == 16 ? 8 : 16);
    if (fmt_csr) return int64_t(P.prow[i]) * q / 4 + i * u;
    return i * (int64_t(P.n / 2) * eb + P.n / 8 + u);
  };
  if (threadIdx.x == 0) {
    int64_t acc = 0;
    for (int p = 0; p < count; ++p) {
      cost0[p] = acc;
      acc += row_cost(probs[p], probs[p].m);
    }
    cost0[count] = acc;
  }
  __syncthreads();
  const int64_t total = cost0[count];
  for (int c = threadIdx.x; c <= slices; c += blockDim.x) {
    if (c == slices) {
      cta_rows[c] = probs[count - 1].row0 + probs[count - 1].m;
      continue;
    }
    const int64_t target = total / slices * c + (total % slices) * c / slices;
    // layer: last p with cost0[p] <= target
    int lo = 0, hi = count - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cost0[mid] <= target) lo = mid; else hi = mid - 1;
    }
    const ApplyProblem& P = probs[lo];
    const int64_t want = target - cost0[lo];
    // first row i in [0, m] with row_cost(i) >= want
    int64_t a = 0, b = P.m;
    while (a < b) {
      const int64_t mid = (a + b) >> 1;
      if (row_cost(P, mid) >= want) b = mid; else a = mid + 1;
    }
    cta_rows[c] = P.row0 + a;
  }
}

}  // namespace

// Slices per SM in a plan; the apply grid (SMs × resident CTAs) divides it for
// every residency 1, 2, 3, 4, 6, 8, 12, 24.
constexpr int kSlicesPerSM = 24;

hsl_status pack_sparse_run(Handle& h, cudaStream_t s) {
  const int eb = dtype_bytes(h.dtype);
  if (h.fmt == HSL_FMT_CSR) {
    const int bits = h.index_bits ? h.index_bits : (h.n < 65535 ? 16 : 32);
    uint32_t* order_flag = static_cast<uint32_t*>(h.err.p) + 1;
    if (cudaError_t e = cudaMemsetAsync(order_flag, 0, 4, s))
      return cuda_fail(e, "column order flag clear");
    if (hsl_status e = ensure(h.prow, size_t(h.m + 1) * 4, "packed row starts")) return e;
    const int64_t grid = std::min<int64_t>((h.m * 32 + 255) / 256, int64_t(h.num_sms) * 8);
    const unsigned tgrid = unsigned(std::max<int64_t>(1, std::min<int64_t>((h.m + 255) / 256,
                                                                          int64_t(h.num_sms) * 8)));
    if (bits == 8) {
      // row lengths with fillers, their padded starts, then the sizes
      if (hsl_status e = ensure(h.d8_lens, size_t(h.m) * 4, "8-bit row lengths")) return e;
      k_csr_d8_len<<<tgrid, 256, 0, s>>>(static_cast<const int32_t*>(h.row_ptr.p),
                                         static_cast<const int32_t*>(h.col.p), h.m, h.nnz,
                                         int32_t(h.n), static_cast<int32_t*>(h.d8_lens.p), order_flag);
      k_csr_prow<<<1, 1024, 0, s>>>(static_cast<const int32_t*>(h.row_ptr.p), h.m, h.nnz,
                                    int64_t(INT32_MAX) & ~int64_t(7), static_cast<int32_t*>(h.prow.p),
                                    static_cast<uint32_t*>(h.err.p),
                                    static_cast<const int32_t*>(h.d8_lens.p));
      note_launch(2);
      int32_t total = 0;
      uint32_t flags = 0;
      if (cudaError_t e = cudaMemcpyAsync(&total, static_cast<int32_t*>(h.prow.p) + h.m, 4,
                                          cudaMemcpyDeviceToHost, s))
        return cuda_fail(e, "8-bit pack size");
      if (cudaError_t e = cudaMemcpyAsync(&flags, order_flag, 4, cudaMemcpyDeviceToHost, s))
        return cuda_fail(e, "8-bit pack size");
      if (cudaError_t e = cudaStreamSynchronize(s)) return cuda_fail(e, "8-bit pack size");
      if (flags & 2u) {
        set_message("8-bit delta columns need the columns of every row in ascending order");
        return HSL_ERR_UNSUPPORTED;
      }
      // slack past the last row: the bulk-fed decode copies whole 64-entry blocks
      const int64_t cap = round_up(int64_t(total) + 64, 64);
      if (hsl_status e = ensure(h.pcol, size_t(cap), "packed column deltas")) return e;
      if (hsl_status e = ensure(h.pbase, size_t(cap / 8) * 2, "packed vector bases")) return e;
      if (hsl_status e = ensure(h.pval, size_t(cap) * eb, "packed values")) return e;
      h.pack_cap = cap;
      if (eb == 2)
        k_csr_d8_fill<uint16_t><<<tgrid, 256, 0, s>>>(
            static_cast<const int32_t*>(h.row_ptr.p), static_cast<const int32_t*>(h.col.p),
            static_cast<const uint16_t*>(h.val.p), static_cast<const int32_t*>(h.prow.p), h.m, h.nnz,
            int32_t(h.n), static_cast<uint8_t*>(h.pcol.p), static_cast<uint16_t*>(h.pbase.p),
            static_cast<uint16_t*>(h.pval.p), static_cast<uint32_t*>(h.err.p));
      else
        k_csr_d8_fill<uint32_t><<<tgrid, 256, 0, s>>>(
            static_cast<const int32_t*>(h.row_ptr.p), static_cast<const int32_t*>(h.col.p),
            static_cast<const uint32_t*>(h.val.p), static_cast<const int32_t*>(h.prow.p), h.m, h.nnz,
            int32_t(h.n), static_cast<uint8_t*>(h.pcol.p), static_cast<uint16_t*>(h.pbase.p),
            static_cast<uint32_t*>(h.pval.p), static_cast<uint32_t*>(h.err.p));
      note_launch();
    } else {
      // every row start a multiple of 8 (16-byte aligned vectors); slack past the
      // last row, as the bulk-fed decode copies whole 64-entry blocks
      const int64_t cap = round_up(h.nnz + 7 * h.m + 64, 64);
      const int cb = bits / 8;
      if (hsl_status e = ensure(h.pcol, size_t(cap) * cb, "packed columns")) return e;
      if (hsl_status e = ensure(h.pval, size_t(cap) * eb, "packed values")) return e;
      h.pack_cap = cap;
      k_csr_prow<<<1, 1024, 0, s>>>(static_cast<const int32_t*>(h.row_ptr.p), h.m, h.nnz, cap,
                                    static_cast<int32_t*>(h.prow.p), static_cast<uint32_t*>(h.err.p),
                                    nullptr);
      note_launch();
      const unsigned g = unsigned(std::max<int64_t>(grid, 1));
      const int32_t* rp = static_cast<const int32_t*>(h.row_ptr.p);
      const int32_t* cl = static_cast<const int32_t*>(h.col.p);
      const int32_t* pr = static_cast<const int32_t*>(h.prow.p);
      uint32_t* err = static_cast<uint32_t*>(h.err.p);
      if (eb == 2 && cb == 2)
        k_csr_fill<uint16_t, uint16_t><<<g, 256, 0, s>>>(rp, cl, static_cast<const uint16_t*>(h.val.p),
            pr, h.m, h.nnz, int32_t(h.n), static_cast<uint16_t*>(h.pcol.p),
            static_cast<uint16_t*>(h.pval.p), err, order_flag);
      else if (eb == 2)
        k_csr_fill<uint16_t, uint32_t><<<g, 256, 0, s>>>(rp, cl, static_cast<const uint16_t*>(h.val.p),
            pr, h.m, h.nnz, int32_t(h.n), static_cast<uint32_t*>(h.pcol.p),
            static_cast<uint16_t*>(h.pval.p), err, order_flag);
      else if (cb == 2)
        k_csr_fill<uint32_t, uint16_t><<<g, 256, 0, s>>>(rp, cl, static_cast<const uint32_t*>(h.val.p),
            pr, h.m, h.nnz, int32_t(h.n), static_cast<uint16_t*>(h.pcol.p),
            static_cast<uint32_t*>(h.pval.p), err, order_flag);
      else
        k_csr_fill<uint32_t, uint32_t><<<g, 256, 0, s>>>(rp, cl, static_cast<const uint32_t*>(h.val.p),
            pr, h.m, h.nnz, int32_t(h.n), static_cast<uint32_t*>(h.pcol.p),
            static_cast<uint32_t*>(h.pval.p), err, order_flag);
      note_launch();
    }
    h.idx_bits = bits;
    // lanes per row: about two 8-entry vectors per lane on an average row
    const double avg_vec = double(h.nnz) / double(std::max<int64_t>(h.m, 1)) / 8.0;
    int g = 4;
    while (g < 32 && g * 2 < avg_vec) g *= 2;
    h.group = g;
    return cuda_fail(cudaGetLastError(), "CSR pack launch");
  }
  // NM24
  if (h.dtype == HSL_BF16 && h.n % 64 == 0) {
    const int64_t tot = ((h.m + 127) / 128) * (h.n / 64) * 128;
    if (hsl_status e = ensure(h.pmeta_tc, size_t(tot) * 8, "2:4 tensor-core metadata")) return e;
    const int64_t g = std::min<int64_t>((tot + 255) / 256, int64_t(h.num_sms) * 16);
    k_meta_tc<<<unsigned(std::max<int64_t>(g, 1)), 256, 0, s>>>(
        static_cast<const uint8_t*>(h.nm_idx.p), h.m, h.n, static_cast<uint2*>(h.pmeta_tc.p));
    note_launch();
  }
  const int64_t nq = (h.n + 15) / 16;  // chunks of 8 kept values per row
  h.meta_stride = int32_t(round_up(nq, 256));
  if (hsl_status e = ensure(h.pmeta, size_t(h.m) * h.meta_stride * 2, "2:4 metadata")) return e;
  const int64_t words = h.m * h.meta_stride;
  const int64_t grid = std::min<int64_t>((words + 255) / 256, int64_t(h.num_sms) * 16);
  k_nm24_meta<<<unsigned(std::max<int64_t>(grid, 1)), 256, 0, s>>>(
      static_cast<const uint8_t*>(h.nm_idx.p), h.m, h.n, h.meta_stride,
      static_cast<uint16_t*>(h.pmeta.p));
  note_launch();
  return cuda_fail(cudaGetLastError(), "2:4 pack launch");
}

hsl_status pack_factors_run(Handle& h, const void* U, const void* V, cudaStream_t s) {
  const int eb = dtype_bytes(h.dtype);
  if (h.r == 0) return HSL_OK;
  if (hsl_status e = ensure(h.U, size_t(h.m) * h.r_pad * eb, "U copy")) return e;
  const int32_t r16 = int32_t(round_up(h.r, 16));
  if (hsl_status e = ensure(h.Vt, size_t(r16) * h.n * eb, "V transpose")) return e;
  const int64_t grid = std::min<int64_t>((h.m * h.r_pad + 255) / 256, int64_t(h.num_sms) * 16);
  const int64_t tgrid =
      std::min<int64_t>(((h.n + 31) / 32) * ((r16 + 31) / 32), int64_t(h.num_sms) * 16);
  if (eb == 2) {
    k_pad_cols<uint16_t><<<unsigned(grid), 256, 0, s>>>(static_cast<const uint16_t*>(U), h.m, h.r,
                                                        h.r_pad, static_cast<uint16_t*>(h.U.p));
    k_transpose_pad<uint16_t><<<unsigned(tgrid), dim3(32, 8), 0, s>>>(
        static_cast<const uint16_t*>(V), h.n, h.r, r16, static_cast<uint16_t*>(h.Vt.p));
  } else {
    k_pad_cols<uint32_t><<<unsigned(grid), 256, 0, s>>>(static_cast<const uint32_t*>(U), h.m, h.r,
                                                        h.r_pad, static_cast<uint32_t*>(h.U.p));
    k_transpose_pad<uint32_t><<<unsigned(tgrid), dim3(32, 8), 0, s>>>(
        static_cast<const uint32_t*>(V), h.n, h.r, r16, static_cast<uint32_t*>(h.Vt.p));
  }
  note_launch(2);
  return cuda_fail(cudaGetLastError(), "factor pack launch");
}

hsl_status plan_build(ApplyPlan& plan, Handle* const* hs, int count, cudaStream_t s) {
  plan.count = count;
  plan.fmt = hs[0]->fmt;
  plan.dtype = hs[0]->dtype;
  plan.n_max = 0;
  plan.r_pad_max = 0;
  plan.vec16 = true;
  plan.err = static_cast<uint32_t*>(hs[0]->err.p);
  plan.idx_bits = hs[0]->idx_bits;
  for (int i = 0; i < count; ++i)
    if (plan.fmt == HSL_FMT_CSR && hs[i]->idx_bits != plan.idx_bits) {
      set_message("a group needs one CSR column width");
      return HSL_ERR_UNSUPPORTED;
    }
  const int eb = dtype_bytes(plan.dtype);
  std::vector<ApplyProblem> probs(count);
  int64_t row0 = 0;
  int zc = 0, zp = 0;
  for (int i = 0; i < count; ++i) {
    Handle& h = *hs[i];
    ApplyProblem& P = probs[i];
    P.prow = static_cast<const int32_t*>(h.prow.p);
    P.pcol = h.pcol.p;
    P.pbase = static_cast<const uint16_t*>(h.pbase.p);
    P.idx_bits = h.idx_bits;
    P.pval = h.fmt == HSL_FMT_CSR ? h.pval.p : h.nm_val.p;
    P.pmeta = static_cast<const uint16_t*>(h.pmeta.p);
    P.U = h.U.p;
    P.Vt = h.Vt.p;
    P.m = int32_t(h.m);
    P.n = int32_t(h.n);
    P.r_pad = h.r_pad;
    P.group = h.group;
    P.meta_stride = h.meta_stride;
    P.row0 = row0;
    row0 += h.m;
    // z = Vᵀx: one work item per row of Vt (a warp each, inside the apply kernel)
    if (h.r_pad > 0)
      if (hsl_status e = ensure(h.z, size_t(16) * h.r_pad * 4, "z")) return e;
    P.z = static_cast<float*>(h.z.p);
    P.z_item0 = zc;
    zc += h.r_pad;
    P.z_piece0 = zp;
    zp += h.r_pad * int32_t((h.n + z_piece_width(int(h.n)) - 1) / z_piece_width(int(h.n)));
    plan.n_max = std::max(plan.n_max, int32_t(h.n));
    plan.vec16 = plan.vec16 && h.n % 16 == 0;
    plan.r_pad_max = std::max(plan.r_pad_max, h.r_pad);
  }
  plan.rows_total = row0;
  plan.z_items = zc;
  plan.z_pieces = zp;
  if (zc > 0 && plan.zsync.p == nullptr) {
    if (hsl_status e = ensure(plan.zsync, 256, "z barrier")) return e;
    if (cudaError_t ce = cudaMemsetAsync(plan.zsync.p, 0, 256, s)) return cuda_fail(ce, "memset");
  }
  const int slices = hs[0]->num_sms * kSlicesPerSM;
  plan.slices = slices;
  if (hsl_status e = ensure(plan.probs, sizeof(ApplyProblem) * count, "plan")) return e;
  if (hsl_status e = ensure(plan.prob_row0, sizeof(int64_t) * (count + 1), "plan")) return e;
  if (hsl_status e = ensure(plan.cta_rows, sizeof(int64_t) * (slices + 1), "plan")) return e;
  std::vector<int64_t> pr0(count + 1);
  for (int i = 0; i < count; ++i) pr0[i] = probs[i].row0;
  pr0[count] = row0;
  if (cudaError_t e = cudaMemcpyAsync(plan.probs.p, probs.data(), sizeof(ApplyProblem) * count,
                                      cudaMemcpyHostToDevice, s))
    return cuda_fail(e, "plan upload");
  if (cudaError_t e = cudaMemcpyAsync(plan.prob_row0.p, pr0.data(), sizeof(int64_t) * (count + 1),
                                      cudaMemcpyHostToDevice, s))
    return cuda_fail(e, "plan upload");
  DevBuf cost0;
  if (hsl_status e = ensure(cost0, sizeof(int64_t) * (count + 1), "plan")) return e;
  k_partition<<<1, 1024, 0, s>>>(static_cast<const ApplyProblem*>(plan.probs.p), count,
                                 plan.fmt == HSL_FMT_CSR ? 1 : 0, eb,
                                 static_cast<int64_t*>(cost0.p), slices,
                                 static_cast<int64_t*>(plan.cta_rows.p));
  note_launch();
  hsl_status st = cuda_fail(cudaGetLastError(), "partition launch");
  // the vectors above are pageable: the copies have completed on return, and
  // the kernel's scratch can be freed once the stream reaches this point
  if (cudaError_t e = cudaStreamSynchronize(s); e != cudaSuccess && st == HSL_OK)
    st = cuda_fail(e, "plan upload");
  release(cost0);
  plan.host_xy.clear();
  return st;
}

}  // namespace hsl
