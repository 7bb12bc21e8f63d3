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
//   2. One emit pass over W, persistent CTAs taking rows in ticket order.  Per
//      row the CTA counts keys > T and keys == T, publishes them, and gets the
//      exclusive prefix over earlier rows by a decoupled look-back (bounded
//      spin; CTAs only wait on rows whose tickets were taken earlier, so they
//      are running).  The row's CSR offset is  gt_before + min(need, eq_before)
//      where need = k − #(key > T): ties are taken in linear order.  A block
//      scan gives each element its rank inside the row; the pass writes the
//      CSR columns/values and the residual (bit copy, +0.0 where kept).
//   HBM traffic: bf16 2 reads of W + 1 write of R + S; fp32 4 reads.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace hsl {
namespace {

struct SelState {
  uint32_t prefix;  // key bits fixed so far (final: the threshold key T)
  uint32_t rem;     // how many still to take among keys matching prefix
  uint32_t gt;      // keys strictly above the prefix range so far
  uint32_t pad;
};

template <typename KT> struct KeyTraits;
template <> struct KeyTraits<uint16_t> {
  static constexpr uint32_t kMask = 0x7FFFu, kInf = 0x7F80u;
};
template <> struct KeyTraits<uint32_t> {
  static constexpr uint32_t kMask = 0x7FFFFFFFu, kInf = 0x7F800000u;
};

__global__ void k_sel_init(SelState* st, uint32_t k, uint32_t prefix) {
  st->prefix = prefix;
  st->rem = k;
  st->gt = 0;
  st->pad = 0;
}

// Histogram of the digit (key >> shift) & (NB-1) over keys whose bits above
// the digit equal st->prefix.
template <typename KT, int BITS>
__global__ void __launch_bounds__(1024) k_split_hist(const KT* __restrict__ W, int64_t count,
                                                     const SelState* __restrict__ st, int shift,
                                                     unsigned* __restrict__ ghist,
                                                     uint32_t* __restrict__ err, int vec_ok) {
  constexpr int NB = 1 << BITS;
  constexpr int EPV = 16 / sizeof(KT);
  extern __shared__ unsigned sh[];
  for (int i = threadIdx.x; i < NB; i += blockDim.x) sh[i] = 0;
  __syncthreads();

  const uint32_t top = uint32_t(shift + BITS);
  const uint32_t hi_mask = top >= 32 ? 0u : (KeyTraits<KT>::kMask & ~((1u << top) - 1u));
  const uint32_t prefix = st->prefix & hi_mask;
  bool nan = false;
  auto one = [&](uint32_t bits) {
    const uint32_t key = bits & KeyTraits<KT>::kMask;
    nan |= key > KeyTraits<KT>::kInf;
    if ((key & hi_mask) == prefix) atomicAdd(&sh[(key >> shift) & (NB - 1)], 1u);
  };

  const int64_t gtid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t gstride = int64_t(gridDim.x) * blockDim.x;
  int64_t done = 0;
  if (vec_ok) {
    const int64_t nvec = count / EPV;
    for (int64_t v = gtid; v < nvec; v += 4 * gstride) {
      uint4 q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t iv = v + u * gstride;
        if (iv < nvec) q[u] = ld_stream16(W + iv * EPV);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (v + u * gstride < nvec) {
          const uint32_t w4[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (sizeof(KT) == 2) {
              one(w4[e] & 0xFFFFu);
              one(w4[e] >> 16);
            } else {
              one(w4[e]);
            }
          }
        }
      }
    }
    done = nvec * EPV;
  }
  for (int64_t e = done + gtid; e < count; e += gstride) one(uint32_t(W[e]));

  if (__syncthreads_or(nan) && threadIdx.x == 0) set_error(err, kErrNaN);
  for (int i = threadIdx.x; i < NB; i += blockDim.x)
    if (sh[i]) atomicAdd(&ghist[i], sh[i]);
}

// One CTA: locate the digit holding the rem-th largest matching key.
__global__ void __launch_bounds__(1024) k_split_select(const unsigned* __restrict__ ghist, int nb,
                                                       int shift, SelState* st) {
  __shared__ unsigned warp_tot[32];
  const int t = threadIdx.x, nt = blockDim.x;
  const int per = (nb + nt - 1) / nt;
  // thread t owns bins [hi - per, hi) counted from the top
  const int hi = nb - t * per, lo = max(0, hi - per);
  unsigned s = 0;
  for (int b = lo; b < hi; ++b) s += ghist[b];
  // exclusive scan over threads (thread 0 = highest bins)
  unsigned incl = s;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
    if ((t & 31) >= o) incl += v;
  }
  if ((t & 31) == 31) warp_tot[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    unsigned w = (t < (nt >> 5)) ? warp_tot[t] : 0u;
    unsigned wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned v = __shfl_up_sync(0xffffffffu, wi, o);
      if (t >= o) wi += v;
    }
    warp_tot[t] = wi - w;  // exclusive warp offsets
  }
  __syncthreads();
  const unsigned before = warp_tot[t >> 5] + incl - s;
  const unsigned rem = st->rem;
  __syncthreads();
  if (rem > before && rem <= before + s) {
    unsigned acc = before;
    for (int b = hi - 1; b >= lo; --b) {
      const unsigned h = ghist[b];
      if (acc + h >= rem) {
        st->gt += acc;
        st->rem = rem - acc;
        st->prefix |= uint32_t(b) << shift;
        break;
      }
      acc += h;
    }
  }
}

// ---- emit -------------------------------------------------------------------
constexpr int kEmitThreads = 256;
constexpr unsigned long long kFlagAgg = 1ull << 62, kFlagInc = 2ull << 62;
constexpr unsigned long long kField = (1ull << 31) - 1;

__device__ __forceinline__ unsigned long long pack_flag(unsigned long long st, uint32_t gt,
                                                        uint32_t eq) {
  return st | ((unsigned long long)gt << 31) | (unsigned long long)eq;
}

template <typename SB> __device__ __forceinline__ SB conv_val(uint32_t bits, int src_bytes);
template <> __device__ __forceinline__ uint16_t conv_val<uint16_t>(uint32_t bits, int src_bytes) {
  if (src_bytes == 2) return uint16_t(bits);
  return __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(bits)));
}
template <> __device__ __forceinline__ uint32_t conv_val<uint32_t>(uint32_t bits, int src_bytes) {
  return src_bytes == 2 ? (bits << 16) : bits;
}

// Block-wide exclusive scan of a packed (gt << 16 | eq) pair; returns the
// exclusive value and writes the block total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* sh_warp,
                                                    uint32_t& total) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sh_warp[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = kEmitThreads / 32;
    uint32_t x = lane < nw ? sh_warp[lane] : 0u;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += u;
    }
    if (lane < nw) sh_warp[lane] = xi - x;
    if (lane == nw - 1) sh_warp[nw] = xi;
  }
  __syncthreads();
  const uint32_t r = sh_warp[w] + incl - v;
  total = sh_warp[kEmitThreads / 32];
  __syncthreads();
  return r;
}

template <typename KT, typename SB>
__global__ void __launch_bounds__(kEmitThreads) k_split_emit(
    const KT* __restrict__ W, int64_t m, int64_t n, const SelState* __restrict__ st,
    unsigned* __restrict__ ticket, unsigned long long* __restrict__ flags,
    int32_t* __restrict__ row_ptr, int32_t* __restrict__ col, SB* __restrict__ val,
    KT* __restrict__ R, int64_t k, uint32_t* __restrict__ err, int vec_ok) {
  constexpr int EPV = 16 / sizeof(KT);
  constexpr int TILE = kEmitThreads * EPV;
  __shared__ uint32_t sh_warp[kEmitThreads / 32 + 1];
  __shared__ uint32_t sh_red[2][kEmitThreads / 32];
  __shared__ int64_t sh_row;
  __shared__ uint32_t sh_excl[2];

  const uint32_t T = st->prefix;
  const uint32_t need = st->rem;
  const int t = threadIdx.x;

  auto load_tile = [&](const KT* rowW, int64_t base, uint32_t (&b)[EPV], bool& valid) {
    const int64_t j0 = base + int64_t(t) * EPV;
    valid = j0 < n;
    if (!valid) return;
    if (vec_ok) {
      const uint4 q = *reinterpret_cast<const uint4*>(rowW + j0);
      const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < EPV; ++e)
        b[e] = sizeof(KT) == 2 ? ((w4[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu) : w4[e];
    } else {
#pragma unroll
      for (int e = 0; e < EPV; ++e) b[e] = (j0 + e < n) ? uint32_t(rowW[j0 + e]) : 0u;
    }
  };

  for (;;) {
    if (t == 0) sh_row = int64_t(atomicAdd(ticket, 1u));
    __syncthreads();
    const int64_t row = sh_row;
    if (row >= m) break;
    const KT* rowW = W + row * n;

    // sweep 1: counts of keys above / equal to T in this row
    uint32_t gt = 0, eq = 0;
    for (int64_t base = 0; base < n; base += TILE) {
      uint32_t b[EPV];
      bool valid;
      load_tile(rowW, base, b, valid);
      if (!valid) continue;
      const int64_t j0 = base + int64_t(t) * EPV;
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        const uint32_t key = b[e] & KeyTraits<KT>::kMask;
        const bool in = j0 + e < n;
        gt += (in && key > T);
        eq += (in && key == T);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if ((t & 31) == 0) {
      sh_red[0][t >> 5] = gt;
      sh_red[1][t >> 5] = eq;
    }
    __syncthreads();
    if (t == 0) {
      uint32_t rg = 0, re = 0;
      for (int w = 0; w < kEmitThreads / 32; ++w) {
        rg += sh_red[0][w];
        re += sh_red[1][w];
      }
      uint32_t xg = 0, xe = 0;
      if (row == 0) {
        st_release_u64(&flags[0], pack_flag(kFlagInc, rg, re));
      } else {
        st_release_u64(&flags[row], pack_flag(kFlagAgg, rg, re));
        int64_t j = row - 1;
        long long spins = 0;
        for (;;) {
          const unsigned long long f = ld_acquire_u64(&flags[j]);
          const unsigned long long s = f & (3ull << 62);
          if (s == 0) {
            if (++spins > kSpinLimit) {
              set_error(err, kErrTimeout);
              break;
            }
            continue;
          }
          xg += uint32_t((f >> 31) & kField);
          xe += uint32_t(f & kField);
          if (s == kFlagInc || j == 0) break;
          --j;
        }
        st_release_u64(&flags[row], pack_flag(kFlagInc, xg + rg, xe + re));
      }
      sh_excl[0] = xg;
      sh_excl[1] = xe;
    }
    __syncthreads();
    const uint32_t ex_gt = sh_excl[0], ex_eq = sh_excl[1];
    const uint32_t taken_before = min(need, ex_eq);
    const int64_t row_start = int64_t(ex_gt) + taken_before;
    if (t == 0) {
      row_ptr[row] = int32_t(row_start);
      if (row == m - 1) row_ptr[m] = int32_t(k);
    }

    // sweep 2: ranks inside the row, CSR entries and the residual
    uint32_t run_gt = 0, run_eq = 0;
    for (int64_t base = 0; base < n; base += TILE) {
      uint32_t b[EPV];
      bool valid;
      load_tile(rowW, base, b, valid);
      const int64_t j0 = base + int64_t(t) * EPV;
      uint32_t lg = 0, le = 0;
      if (valid) {
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
          const uint32_t key = b[e] & KeyTraits<KT>::kMask;
          const bool in = j0 + e < n;
          lg += (in && key > T);
          le += (in && key == T);
        }
      }
      uint32_t tot;
      const uint32_t ex = block_excl_scan((lg << 16) | le, sh_warp, tot);
      uint32_t cg = run_gt + (ex >> 16), ce = run_eq + (ex & 0xFFFFu);
      if (valid) {
        uint32_t rb[EPV];
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
          const uint32_t key = b[e] & KeyTraits<KT>::kMask;
          const bool in = j0 + e < n;
          const bool g = in && key > T;
          const bool q = in && key == T;
          const bool sel = g || (q && (ex_eq + ce) < need);
          if (sel) {
            const uint32_t before = cg + (min(need, ex_eq + ce) - taken_before);
            const int64_t pos = row_start + before;
            if (pos < k) {
              col[pos] = int32_t(j0 + e);
              val[pos] = conv_val<SB>(b[e], sizeof(KT));
            }
          }
          rb[e] = sel ? 0u : b[e];
          cg += g;
          ce += q;
        }
        if (vec_ok) {
          uint4 o;
          if (sizeof(KT) == 2) {
            o.x = rb[0] | (rb[1 % EPV] << 16);
            o.y = rb[2 % EPV] | (rb[3 % EPV] << 16);
            o.z = rb[4 % EPV] | (rb[5 % EPV] << 16);
            o.w = rb[6 % EPV] | (rb[7 % EPV] << 16);
          } else {
            o.x = rb[0];
            o.y = rb[1 % EPV];
            o.z = rb[2 % EPV];
            o.w = rb[3 % EPV];
          }
          if (R) *reinterpret_cast<uint4*>(R + row * n + j0) = o;
        } else if (R) {
#pragma unroll
          for (int e = 0; e < EPV; ++e)
            if (j0 + e < n) R[row * n + j0 + e] = KT(rb[e]);
        }
      }
      run_gt += tot >> 16;
      run_eq += tot & 0xFFFFu;
    }
  }
}

template <typename KT, typename SB>
hsl_status emit_launch(Handle& h, const KT* W, int64_t k, KT* R, SelState* st, unsigned* ticket,
                       unsigned long long* flags, uint32_t* err, bool vec_ok, cudaStream_t s) {
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
