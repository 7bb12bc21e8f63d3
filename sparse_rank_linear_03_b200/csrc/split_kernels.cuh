// Device code of the magnitude top-k split (see split_topk.cu for the design):
// radix-digit histogram, digit select, and the two emit kernels (row tickets;
// blocks of rows held in registers).  Included by the .cu files that launch
// them; everything here has internal linkage.
#pragma once

#include "common.cuh"

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

// ---- emit over blocks of rows held in registers ---------------------------------
// A CTA takes a ticket for `rb` consecutive rows (rb·n ≤ 256·kVPT·EPV elements),
// loads them once into registers (coalesced 16-byte vectors, vector v of the
// block at k-major position v = kk·256 + t), ranks every element inside the
// block with warp scans per kk plus one scan of the (kk, warp) totals, and
// gets the block's exclusive prefix by a warp-parallel decoupled look-back
// (32 predecessor flags per poll).
constexpr int kVPT = 16;

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// Warp 0 only.  Publishes the block aggregate, returns the exclusive prefix.
__device__ __forceinline__ void lookback(unsigned long long* flags, int64_t blk, uint32_t agg_gt,
                                         uint32_t agg_eq, uint32_t* err, uint32_t& ex_gt,
                                         uint32_t& ex_eq) {
  const int lane = threadIdx.x & 31;
  if (blk == 0) {
    if (lane == 0) st_release_u64(&flags[0], pack_flag(kFlagInc, agg_gt, agg_eq));
    ex_gt = ex_eq = 0;
    return;
  }
  if (lane == 0) st_release_u64(&flags[blk], pack_flag(kFlagAgg, agg_gt, agg_eq));
  uint32_t xg = 0, xe = 0;
  int64_t base = blk - 1;
  long long spins = 0;
  for (;;) {
    const int64_t j = base - lane;
    const unsigned long long f = j >= 0 ? ld_acquire_u64(&flags[j]) : kFlagInc;  // before block 0
    const unsigned long long s = f & (3ull << 62);
    const unsigned inc = __ballot_sync(0xffffffffu, s == kFlagInc);
    const unsigned notready = __ballot_sync(0xffffffffu, s == 0);
    const int first = inc ? __ffs(inc) - 1 : 32;
    const unsigned needed = first >= 31 ? 0xffffffffu : ((2u << first) - 1u);
    if (notready & needed) {
      if (++spins > kSpinLimit) {
        if (lane == 0) set_error(err, kErrTimeout);
        break;
      }
      continue;
    }
    uint32_t g = 0, e = 0;
    if (lane <= first) {
      g = uint32_t((f >> 31) & kField);
      e = uint32_t(f & kField);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    xg += g;
    xe += e;
    if (first < 32) break;
    base -= 32;
  }
  ex_gt = xg;
  ex_eq = xe;
  if (lane == 0) st_release_u64(&flags[blk], pack_flag(kFlagInc, xg + agg_gt, xe + agg_eq));
}

// Masks of one 16-byte vector: bit e = element e has key > T (gm) / key == T (em).
// bf16: two 15-bit keys per word, compared without branches by one packed
// subtraction per threshold: with k' = key | 0x8000 in each half and t ≤ 0x8000,
// bit 15 of (k' − t) is set iff key ≥ t, and no half ever borrows from the next.
template <typename KT>
__device__ __forceinline__ void vec_masks(const uint4& q, uint32_t T, uint32_t& gm, uint32_t& em);
template <>
__device__ __forceinline__ void vec_masks<uint16_t>(const uint4& q, uint32_t T, uint32_t& gm,
                                                    uint32_t& em) {
  const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
  const uint32_t T0 = T <= 0x7FFFu ? T : 0x8000u;  // T above every key: nothing ≥ T
  const uint32_t TT = T0 * 0x00010001u, TT1 = (T0 + 1u) * 0x00010001u;
  uint32_t ge = 0, gt = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t k = (w4[u] & 0x7FFF7FFFu) | 0x80008000u;
    const uint32_t a = (k - TT) & 0x80008000u;
    const uint32_t b = T0 >= 0x7FFFu ? 0u : ((k - TT1) & 0x80008000u);
    ge |= (((a >> 15) | (a >> 30)) & 3u) << (2 * u);
    gt |= (((b >> 15) | (b >> 30)) & 3u) << (2 * u);
  }
  gm = gt;
  em = ge & ~gt;
}
template <>
__device__ __forceinline__ void vec_masks<uint32_t>(const uint4& q, uint32_t T, uint32_t& gm,
                                                    uint32_t& em) {
  const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
  gm = em = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t k = w4[u] & 0x7FFFFFFFu;
    gm |= uint32_t(k > T) << u;
    em |= uint32_t(k == T) << u;
  }
}

template <typename KT, typename SB>
__global__ void __launch_bounds__(kEmitThreads) k_split_emit_blk(
    const KT* __restrict__ W, int64_t m, int64_t n, int rb, int64_t nblk,
    const SelState* __restrict__ st, unsigned* __restrict__ ticket,
    unsigned long long* __restrict__ flags, int32_t* __restrict__ row_ptr,
    int32_t* __restrict__ col, SB* __restrict__ val, KT* __restrict__ R, int64_t k,
    uint32_t* __restrict__ err) {
  constexpr int EPV = 16 / sizeof(KT);
  constexpr uint32_t STEP = kEmitThreads * EPV;  // elements between a thread's vectors
  __shared__ uint32_t wt[kVPT][kEmitThreads / 32];
  __shared__ int64_t sh_blk;
  __shared__ uint32_t sh_ex[2];
  const uint32_t T = st->prefix;
  const uint32_t need = st->rem;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint32_t n32 = uint32_t(n);

  for (;;) {
    if (t == 0) sh_blk = int64_t(atomicAdd(ticket, 1u));
    __syncthreads();
    const int64_t blk = sh_blk;
    if (blk >= nblk) break;
    const int64_t row0 = blk * rb;
    const int64_t rows = min(int64_t(rb), m - row0);
    const int64_t e0 = row0 * n;
    const uint32_t nv = uint32_t(rows * n / EPV);
    const KT* Wb = W + e0;

    // phase 1: load the block (coalesced, k-major), masks, ranks inside the block
    uint4 q[kVPT];
    uint32_t ex[kVPT];
    uint32_t mk[kVPT / 2];  // (gm | em << 8) of vector kk in half kk & 1
#pragma unroll
    for (int kk = 0; kk < kVPT; ++kk) {
      const uint32_t v = uint32_t(kk * kEmitThreads + t);
      uint32_t pk = 0, gm = 0, em = 0;
      if (v < nv) {
        q[kk] = ld_stream16(Wb + int64_t(v) * EPV);
        vec_masks<KT>(q[kk], T, gm, em);
        pk = (uint32_t(__popc(gm)) << 16) | uint32_t(__popc(em));
      }
      const uint32_t m16 = gm | (em << 8);
      if (kk & 1) mk[kk >> 1] |= m16 << 16; else mk[kk >> 1] = m16;
      const uint32_t incl = warp_incl_scan(pk);
      ex[kk] = incl - pk;
      if (lane == 31) wt[kk][warp] = incl;
    }
    __syncthreads();
    if (warp == 0) {
      // exclusive scan of the kVPT × 8 totals in k-major order: lane takes 4
      uint32_t a[4], local = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = 4 * lane + u;
        a[u] = wt[idx >> 3][idx & 7];
        local += a[u];
      }
      const uint32_t incl = warp_incl_scan(local);
      uint32_t run = incl - local;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = 4 * lane + u;
        wt[idx >> 3][idx & 7] = run;
        run += a[u];
      }
      const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
      uint32_t xg, xe;
      lookback(flags, blk, total >> 16, total & 0xFFFFu, err, xg, xe);
      if (lane == 0) {
        sh_ex[0] = xg;
        sh_ex[1] = xe;
      }
    }
    __syncthreads();
    // phase 2: kept before an element = keys > T before it + the first `need`
    // ties in linear order that come before it
    const uint32_t ex_gt = sh_ex[0], ex_eq = sh_ex[1];
    uint32_t j0 = uint32_t(t) * EPV;  // column of this thread's first vector, no division
    int64_t row = row0;
    while (j0 >= n32) {
      j0 -= n32;
      ++row;
    }
#pragma unroll
    for (int kk = 0; kk < kVPT; ++kk) {
      const uint32_t v = uint32_t(kk * kEmitThreads + t);
      if (v < nv) {
        const uint32_t m16 = (mk[kk >> 1] >> ((kk & 1) * 16)) & 0xFFFFu;
        const uint32_t gm = m16 & 0xFFu, em = m16 >> 8;
        const uint32_t base = wt[kk][warp] + ex[kk];
        const uint32_t cg = base >> 16, ce = base & 0xFFFFu;
        const uint32_t pos0 = ex_gt + cg + min(need, ex_eq + ce);
        if (j0 == 0) row_ptr[row] = int32_t(pos0);
        // ties kept in this vector: the first `allow` set bits of em
        uint32_t allow = need > ex_eq + ce ? min(need - (ex_eq + ce), uint32_t(__popc(em))) : 0u;
        uint32_t keq = 0, rest = em;
        for (; allow; --allow) {
          keq |= rest & (0u - rest);
          rest &= rest - 1u;
        }
        const uint32_t sel = gm | keq;
        uint4 o = q[kk];
        if (sel) {
          for (uint32_t s2 = sel; s2; s2 &= s2 - 1u) {
            const int e = __ffs(s2) - 1;
            const int64_t pos = int64_t(pos0) + __popc(sel & ((1u << e) - 1u));
            const uint32_t w = (&o.x)[sizeof(KT) == 2 ? (e >> 1) : e];
            const uint32_t bits = sizeof(KT) == 2 ? ((w >> ((e & 1) * 16)) & 0xFFFFu) : w;
            if (pos < k) {
              col[pos] = int32_t(j0 + e);
              val[pos] = conv_val<SB>(bits, sizeof(KT));
            }
          }
          // zero the kept elements in the residual
          uint32_t* ow = &o.x;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t z;
            if (sizeof(KT) == 2)
              z = (((sel >> (2 * u)) & 1u) ? 0x0000FFFFu : 0u) |
                  (((sel >> (2 * u + 1)) & 1u) ? 0xFFFF0000u : 0u);
            else
              z = ((sel >> u) & 1u) ? 0xFFFFFFFFu : 0u;
            ow[u] &= ~z;
          }
        }
        if (R) st_stream16(R + e0 + int64_t(v) * EPV, o);
      }
      j0 += STEP;
      while (j0 >= n32) {
        j0 -= n32;
        ++row;
      }
    }
    if (t == 0 && blk == nblk - 1) row_ptr[m] = int32_t(k);
  }
}

}  // namespace
}  // namespace hsl
