// Device code of the magnitude top-k split (see split_topk.cu for the design):
// the sampled bracket (sample histogram, bracket select, count pass, finish,
// per-tile counts and their scan), the radix-digit histogram and digit
// select, and the two emit kernels (k_split_emit: one row per ticket;
// k_split_emit_tile: tiles staged in shared memory by bulk copies).  Included
// by the .cu files that launch them; everything here has internal linkage.
#pragma once

#include "common.cuh"
#include "tc.cuh"

namespace hsl {
namespace {

struct SelState {
  uint32_t prefix;  // key bits fixed so far (final: the threshold key T)
  uint32_t rem;     // how many still to take among keys matching prefix
  uint32_t gt;      // keys strictly above the prefix range so far
  uint32_t pad;
};

// Emit tiles: W is processed in tiles of TB bytes by CTAs of kTileThreads.
// Tiles whose S prefixes come from the bracket pass's per-tile counts are
// small, so four CTAs share an SM and hide each other's per-tile latency;
// tiles that find their prefix by look-back are twice as large, which halves
// the number of look-backs.
constexpr int kTileThreads = 256;
constexpr int kTileBytesPre = 16384;
constexpr int kTileBytesLB = 32768;
constexpr int kStages = 3;
// The emit refills, at the end of iteration it, the stage that iteration
// it + kStages - 1 consumes, and writes that stage's tile id there too: the
// barriers of the iterations in between make the id visible to every thread.
// With two stages the next iteration would read the id before any barrier.
static_assert(kStages >= 3, "the emit's tile ids need three stages");

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
                                                     uint32_t* __restrict__ err, int vec_ok,
                                                     const uint32_t* __restrict__ skip) {
  if (skip && *skip) return;  // the threshold is already known
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
                                                       int shift, SelState* st,
                                                       const uint32_t* __restrict__ skip) {
  if (skip && *skip) return;
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

// The eight flags at bits 15 / 31 of four words (element 2u / 2u + 1 of word
// u) as an 8-bit mask in element order: one byte permute per word pair puts
// the flags at the top bit of each byte, and a multiply by 2^0 + 2^7 + 2^14 +
// 2^21 gathers the four byte-top bits into bits 28..31 (no two partial
// products meet, so nothing carries).
__device__ __forceinline__ uint32_t gather_flags8(const uint32_t (&f)[4]) {
  const uint32_t lo = __byte_perm(f[0], f[1], 0x7531), hi = __byte_perm(f[2], f[3], 0x7531);
  return ((lo * 0x00204081u) >> 28) | (((hi * 0x00204081u) >> 24) & 0xF0u);
}
// ---- bf16 threshold from a sampled bracket ------------------------------------
// A sample of W (one run of kSampleRun vectors at a hashed offset in every
// stratum of kSampleStride vectors) brackets the key of the k-th largest
// magnitude: [lo, hi] around the sample's rank k·S/count with a wide margin.
// One pass over W then counts keys > hi and histograms only the keys inside
// the bracket (a few percent of W), replacing a shared-memory atomic per
// element by two packed compares.  If the true threshold is not inside the
// bracket (the sample misled), the full histogram pass runs instead; the
// result is exact either way.
constexpr int kSampleRun = 32;        // vectors of 8 bf16 per sampled run
constexpr int kSampleStride = 2048;   // vectors per stratum (one run each)

struct Bracket {
  uint32_t lo, hi;  // keys in [lo, hi] are histogrammed, keys > hi counted
  uint32_t above;   // number of keys > hi
  uint32_t ok;      // 1 when the threshold was found inside the bracket
};

__device__ __forceinline__ uint32_t mix32(uint32_t x) {  // integer hash (lowbias32)
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}

// Histogram of the sampled 15-bit keys (NaN keys left out).
__global__ void __launch_bounds__(1024) k_sample_hist(const uint16_t* __restrict__ W,
                                                      int64_t nstrata,
                                                      unsigned* __restrict__ shist) {
  extern __shared__ unsigned sh[];
  for (int i = threadIdx.x; i < 32768; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t c = gw; c < nstrata; c += nw) {  // one warp per run, a vector per lane
    const int64_t v0 = c * kSampleStride + mix32(uint32_t(c)) % uint32_t(kSampleStride - kSampleRun + 1);
    const uint4 q = ld_stream16(W + (v0 + lane) * 8);
    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t k0 = w4[u] & 0x7FFFu, k1 = (w4[u] >> 16) & 0x7FFFu;
      if (k0 <= 0x7F80u) atomicAdd(&sh[k0], 1u);
      if (k1 <= 0x7F80u) atomicAdd(&sh[k1], 1u);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 32768; i += blockDim.x)
    if (sh[i]) atomicAdd(&shist[i], sh[i]);
}

// One CTA: per thread 32 bins counted from the top key down; returns through
// `rank_key` the key at which the inclusive count from the top first reaches
// each target rank (lo for r_lo, hi for r_hi).
__global__ void __launch_bounds__(1024) k_bracket_select(const unsigned* __restrict__ shist,
                                                         uint32_t r_hi, uint32_t r_lo,
                                                         Bracket* __restrict__ br) {
  __shared__ unsigned warp_tot[32];
  __shared__ uint32_t key_hi, key_lo;
  const int t = threadIdx.x;
  constexpr int PER = 32768 / 1024;
  if (t == 0) {
    key_hi = 0x7FFFu;  // r_hi == 0: nothing is certainly above the threshold
    key_lo = 0u;       // r_lo beyond the sample: keep every key in the bracket
  }
  const int top = 32767 - t * PER;  // this thread's bins: top, top−1, ..., top−PER+1
  // the 32 bins [top − 31, top] are one aligned 128-byte run: eight 16-byte loads
  unsigned hb[PER];
  {
    const uint4* src = reinterpret_cast<const uint4*>(shist + (top - PER + 1));
#pragma unroll
    for (int u = 0; u < PER / 4; ++u) {
      const uint4 q = src[u];
      hb[4 * u] = q.x;
      hb[4 * u + 1] = q.y;
      hb[4 * u + 2] = q.z;
      hb[4 * u + 3] = q.w;
    }
  }
  unsigned s = 0;
#pragma unroll
  for (int b = 0; b < PER; ++b) s += hb[b];
  unsigned incl = s;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
    if ((t & 31) >= o) incl += v;
  }
  if ((t & 31) == 31) warp_tot[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    const unsigned w = warp_tot[t];
    unsigned wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned v = __shfl_up_sync(0xffffffffu, wi, o);
      if (t >= o) wi += v;
    }
    warp_tot[t] = wi - w;
  }
  __syncthreads();
  const unsigned before = warp_tot[t >> 5] + incl - s;
  // hi: the largest key with more than r_hi sample keys at or above it, so at
  // most r_hi sample keys lie strictly above hi
  if (r_hi > 0 && r_hi >= before && r_hi < before + s) {
    unsigned acc = before;
    for (int b = 0; b < PER; ++b) {
      acc += hb[PER - 1 - b];  // bin top − b
      if (acc > r_hi) {
        key_hi = uint32_t(top - b);
        break;
      }
    }
  }
  // lo: the largest key with at least r_lo sample keys at or above it
  if (r_lo > before && r_lo <= before + s) {
    unsigned acc = before;
    for (int b = 0; b < PER; ++b) {
      acc += hb[PER - 1 - b];
      if (acc >= r_lo) {
        key_lo = uint32_t(top - b);
        break;
      }
    }
  }
  __syncthreads();
  if (t == 0) {
    br->hi = key_hi;
    br->lo = min(key_lo, key_hi);
    br->above = 0;
    br->ok = 0;
  }
}

// Full pass: count keys > hi, histogram keys in [lo, hi] into ghist[key],
// flag NaN.  bf16 pairs are compared by packed subtraction (see vec_masks).
// When the bracket spans at most kTileBins keys and tile_hist is given, each
// warp takes whole emit tiles (kTileBytesPre of W) and also records, per tile,
// the count above the bracket and the tile's bracket histogram; with the
// threshold known, those give every tile's exact (above T, equal to T) counts,
// so the emit pass needs no look-back.
constexpr int kTileBins = 64;

__global__ void __launch_bounds__(1024) k_count_bracket(const uint16_t* __restrict__ W,
                                                        int64_t nvec, Bracket* __restrict__ br,
                                                        unsigned* __restrict__ ghist,
                                                        uint32_t* __restrict__ err,
                                                        uint32_t* __restrict__ tile_above,
                                                        uint32_t* __restrict__ tile_hist) {
  extern __shared__ unsigned sh[];
  __shared__ unsigned warp_above[32];
  __shared__ unsigned wh[32][kTileBins];
  const uint32_t lo = br->lo, hi = br->hi;
  const int nb = int(hi - lo) + 1;
  const bool record = tile_hist != nullptr && nb <= kTileBins;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) sh[i] = 0;
  for (int i = lane; i < kTileBins; i += 32) wh[warp][i] = 0;
  __syncthreads();
  unsigned* bins = record ? wh[warp] : sh;
  const uint32_t H = 0x80008000u;
  const uint32_t HI1 = (hi + 1u) * 0x00010001u, LO = lo * 0x00010001u, NAN1 = 0x7F81u * 0x00010001u;
  unsigned above = 0;
  uint32_t nan = 0;  // bit 15 / 31 set once some key ≥ 0x7F81 (a NaN)
  // one 16-byte vector: keys above hi add to two 16-bit counters in `cnt`
  // (flushed by the caller before either could reach 2^16), keys inside the
  // bracket (rare) go to the histogram
  auto vec = [&](const uint4& q, uint32_t& cnt) {
    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
    uint32_t in4[4], any = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t kw = w4[u] | H;
      const uint32_t dh = kw - HI1;
      nan |= kw - NAN1;
      cnt += (dh & H) >> 15;
      in4[u] = (kw - LO) & ~dh & H;
      any |= in4[u];
    }
    if (any) {  // usually one element of the lane: walk the set bits
      for (uint32_t mk = gather_flags8(in4); mk; mk &= mk - 1u) {
        const int e = __ffs(mk) - 1;
        const uint32_t w = (e & 4) ? ((e & 2) ? w4[3] : w4[2]) : ((e & 2) ? w4[1] : w4[0]);
        atomicAdd(&bins[((w >> ((e & 1) * 16)) & 0x7FFFu) - lo], 1u);
      }
    }
  };
  auto flush = [&](uint32_t& cnt) {
    above += (cnt & 0xFFFFu) + (cnt >> 16);
    cnt = 0;
  };
  if (record) {
    constexpr int VPT = kTileBytesPre / 16;  // vectors of a tile
    const int64_t ntiles = (nvec + VPT - 1) / VPT;
    const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
    unsigned above_all = 0;
    for (int64_t tile = gw; tile < ntiles; tile += nw) {
      const int64_t v0 = tile * VPT, vend = min(v0 + VPT, nvec);
      above = 0;
      uint32_t cnt = 0;  // ≤ 64 vectors · 4 words per lane and tile: no overflow
      for (int it = 0; it < VPT / 32; it += 8) {
        uint4 q[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t v = v0 + (it + u) * 32 + lane;
          if (v < vend) q[u] = ld_stream16(W + v * 8);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (v0 + (it + u) * 32 + lane < vend) vec(q[u], cnt);
      }
      flush(cnt);
      for (int o = 16; o; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
      __syncwarp();
      for (int b = lane; b < kTileBins; b += 32) {
        const unsigned c = wh[warp][b];
        tile_hist[tile * kTileBins + b] = c;
        if (c) atomicAdd(&sh[b], c);
        wh[warp][b] = 0;
      }
      if (lane == 0) tile_above[tile] = above;
      above_all += above;
      __syncwarp();
    }
    above = lane == 0 ? above_all : 0u;
  } else {
    const int64_t gtid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t gstride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t v = gtid; v < nvec; v += 4 * gstride) {
      uint4 q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t iv = v + u * gstride;
        if (iv < nvec) q[u] = ld_stream16(W + iv * 8);
      }
      uint32_t cnt = 0;  // 16 words at most before the flush
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (v + u * gstride < nvec) vec(q[u], cnt);
      flush(cnt);
    }
  }
  for (int o = 16; o; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
  if (lane == 0) warp_above[warp] = above;
  if (__syncthreads_or((nan & H) != 0) && threadIdx.x == 0) set_error(err, kErrNaN);
  if (threadIdx.x == 0) {
    unsigned a = 0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) a += warp_above[w];
    atomicAdd(&br->above, a);
  }
  for (int i = threadIdx.x; i < nb; i += blockDim.x)
    if (sh[i]) atomicAdd(&ghist[lo + i], sh[i]);
}

// Whether the tile counts recorded by k_count_bracket give the emit its
// prefixes: the bracket held the threshold and was narrow enough to record.
__device__ __forceinline__ bool tile_counts_usable(const Bracket* br) {
  return br->ok && br->hi - br->lo + 1u <= uint32_t(kTileBins);
}

// Per tile: (keys > T) << 32 | (keys == T), one warp per tile.
__global__ void __launch_bounds__(256) k_tile_counts(const uint32_t* __restrict__ tile_above,
                                                     const uint32_t* __restrict__ tile_hist,
                                                     int64_t ntiles, const Bracket* __restrict__ br,
                                                     const SelState* __restrict__ st,
                                                     unsigned long long* __restrict__ tile_cnt) {
  if (!tile_counts_usable(br)) return;
  const uint32_t T = st->prefix, lo = br->lo;
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  constexpr int TW = 4;  // tiles per warp at a time: eight loads in flight per lane
  for (int64_t tile0 = gw * TW; tile0 < ntiles; tile0 += nw * TW) {
    unsigned c[TW][2];
#pragma unroll
    for (int u = 0; u < TW; ++u)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        c[u][h] = tile0 + u < ntiles ? tile_hist[(tile0 + u) * kTileBins + lane + 32 * h] : 0u;
#pragma unroll
    for (int u = 0; u < TW; ++u) {
      unsigned gt = 0, eq = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t key = lo + uint32_t(lane + 32 * h);
        gt += key > T ? c[u][h] : 0u;
        eq += key == T ? c[u][h] : 0u;
      }
      for (int o = 16; o; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
      }
      if (lane == 0 && tile0 + u < ntiles)
        tile_cnt[tile0 + u] = ((unsigned long long)(tile_above[tile0 + u] + gt) << 32) | eq;
    }
  }
}

// One CTA: exclusive prefix of the packed tile counts (both halves stay below
// 2^32 because W has fewer than 2^32 elements on this path).
__global__ void __launch_bounds__(1024) k_tile_scan(const unsigned long long* __restrict__ tile_cnt,
                                                    int64_t ntiles, const Bracket* __restrict__ br,
                                                    unsigned long long* __restrict__ tile_pre) {
  if (!tile_counts_usable(br)) return;
  __shared__ unsigned long long warp_tot[32];
  const int t = threadIdx.x;
  const int64_t per = (ntiles + 1023) / 1024;
  const int64_t a = min(int64_t(t) * per, ntiles), b = min(a + per, ntiles);
  constexpr int RB = 16;  // up to 16 tiles per thread are loaded at once and kept
  unsigned long long reg[RB];
  unsigned long long s = 0;
  if (per <= RB) {
#pragma unroll
    for (int u = 0; u < RB; ++u) reg[u] = a + u < b ? tile_cnt[a + u] : 0ull;
#pragma unroll
    for (int u = 0; u < RB; ++u) s += reg[u];
  } else {
    for (int64_t i = a; i < b; ++i) s += tile_cnt[i];
  }
  unsigned long long incl = s;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if ((t & 31) >= o) incl += v;
  }
  if ((t & 31) == 31) warp_tot[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    const unsigned long long w = warp_tot[t];
    unsigned long long wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long v = __shfl_up_sync(0xffffffffu, wi, o);
      if (t >= o) wi += v;
    }
    warp_tot[t] = wi - w;
  }
  __syncthreads();
  unsigned long long run = warp_tot[t >> 5] + incl - s;
  if (per <= RB) {
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      if (a + u < b) tile_pre[a + u] = run;
      run += reg[u];
    }
  } else {
    for (int64_t i = a; i < b; ++i) {
      tile_pre[i] = run;
      run += tile_cnt[i];
    }
  }
}

// One CTA: the threshold from the bracket, or (threshold outside it) a clean
// state and histogram for the full pass.
__global__ void __launch_bounds__(1024) k_bracket_finish(unsigned* __restrict__ ghist,
                                                         Bracket* __restrict__ br,
                                                         SelState* __restrict__ st, uint32_t k) {
  __shared__ unsigned warp_tot[32];
  __shared__ int found;
  const int t = threadIdx.x;
  const uint32_t lo = br->lo, hi = br->hi, above = br->above;
  const int nb = int(hi - lo) + 1;
  const int per = (nb + 1023) / 1024;
  if (t == 0) found = 0;
  const int top = int(hi) - t * per;  // bins top, top−1, ... (≥ lo)
  unsigned s = 0;
  for (int b = 0; b < per; ++b)
    if (top - b >= int(lo)) s += ghist[top - b];
  unsigned incl = s;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
    if ((t & 31) >= o) incl += v;
  }
  if ((t & 31) == 31) warp_tot[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    const unsigned w = warp_tot[t];
    unsigned wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned v = __shfl_up_sync(0xffffffffu, wi, o);
      if (t >= o) wi += v;
    }
    warp_tot[t] = wi - w;
  }
  __syncthreads();
  const unsigned before = above + warp_tot[t >> 5] + incl - s;
  if (k > before && k <= before + s) {
    unsigned acc = before;
    for (int b = 0; b < per && top - b >= int(lo); ++b) {
      const unsigned h = ghist[top - b];
      if (acc + h >= k) {
        st->prefix = uint32_t(top - b);
        st->rem = k - acc;
        st->gt = acc;
        found = 1;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
  if (t == 0) br->ok = uint32_t(found);
  if (!found) {  // back to the state the full histogram pass expects
    for (int i = t; i < nb; i += 1024) ghist[lo + i] = 0;
    if (t == 0) {
      st->prefix = 0;
      st->rem = k;
      st->gt = 0;
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

// Block-wide exclusive scan with two barriers: the warp totals go to one of
// two buffers (alternate calls use the other), so no third barrier is needed
// before the buffer is written again.
__device__ __forceinline__ uint32_t block_excl_scan2(uint32_t v, uint32_t (*sh)[kEmitThreads / 32 + 1],
                                                     int parity, uint32_t& total) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  uint32_t* sw = sh[parity];
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sw[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = kEmitThreads / 32;
    uint32_t x = lane < nw ? sw[lane] : 0u;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += u;
    }
    if (lane < nw) sw[lane] = xi - x;
    if (lane == nw - 1) sw[nw] = xi;
  }
  __syncthreads();
  total = sw[kEmitThreads / 32];
  return sw[w] + incl - v;
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
  uint32_t a[4], b[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t k = w4[u] | 0x80008000u;
    a[u] = (k - TT) & 0x80008000u;
    b[u] = T0 >= 0x7FFFu ? 0u : ((k - TT1) & 0x80008000u);
  }
  const uint32_t ge = gather_flags8(a);
  gm = gather_flags8(b);
  em = ge & ~gm;
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

// ---- emit over element tiles staged by bulk copies -----------------------------
// W is cut into tiles of TB bytes (any number of rows or part of one).  A
// persistent CTA takes tiles in ticket order and keeps kStages of them in
// flight: a 1-D bulk copy brings each into shared memory; the residual goes
// back with a bulk store from the same buffer.  Thread t owns TB / 4096
// contiguous vectors of its tile and starts at a slot chosen so that, at every
// step, the eight threads of a quarter-warp read eight different bank groups.
// The kept entries of a tile form a contiguous range of S; after one barrier
// every thread produces outputs i, i + 256, ... of that range (binary search
// for the owning thread, then its (i − first)-th kept element), so S is
// written with coalesced stores and the kept elements are zeroed in the staged
// tile, which the bulk store writes back as the residual.

// Unsigned 32-bit division by an invariant divisor d (1 ≤ d < 2^31): with
// l = ceil(log2 d) and mult = floor(2^32·(2^l − d)/d) + 1,
// q = (t + ((x − t) >> s1)) >> s2, t = mulhi(mult, x), s1 = min(l, 1),
// s2 = max(l − 1, 0), exact for every 32-bit x (Granlund & Montgomery 1994).
struct FastDiv {
  uint32_t d, mult, s1, s2;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t l = 0;
  while ((uint64_t(1) << l) < d) ++l;
  f.mult = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1);
  f.s1 = l < 1 ? l : 1;
  f.s2 = l > 1 ? l - 1 : 0;
  return f;
}
__device__ __forceinline__ uint32_t fdiv(const FastDiv& f, uint32_t x) {
  const uint32_t t = __umulhi(f.mult, x);
  return (t + ((x - t) >> f.s1)) >> f.s2;
}

// Index of the j-th set bit (j counted from 0) of m; m has more than j set bits.
__device__ __forceinline__ int nth_set_bit64(unsigned long long m, uint32_t j) {
  uint32_t w = uint32_t(m);
  int base = 0;
  uint32_t c = uint32_t(__popc(w));
  if (j >= c) {
    j -= c;
    w = uint32_t(m >> 32);
    base = 32;
  }
#pragma unroll
  for (int half = 16; half; half >>= 1) {
    c = uint32_t(__popc(w & ((1u << half) - 1u)));
    if (j >= c) {
      j -= c;
      w >>= half;
      base += half;
    }
  }
  return base;
}

template <typename KT, typename SB, int TB>
__global__ void __launch_bounds__(kTileThreads, TB <= 16384 ? 4 : 2) k_split_emit_tile(
    const KT* __restrict__ W, int64_t m, int64_t count, FastDiv nd, int64_t ntiles,
    const SelState* __restrict__ st, unsigned* __restrict__ ticket,
    unsigned long long* __restrict__ flags, int32_t* __restrict__ row_ptr,
    int32_t* __restrict__ col, SB* __restrict__ val, KT* __restrict__ R, int64_t k,
    uint32_t* __restrict__ err, const Bracket* __restrict__ br,
    const unsigned long long* __restrict__ tile_pre) {
  constexpr int EPV = 16 / sizeof(KT);
  constexpr int TE = TB / sizeof(KT);
  constexpr int kTileVPT = TB / 16 / kTileThreads;  // vectors per thread
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* tiles = reinterpret_cast<uint4*>(smem);
  __shared__ unsigned long long s_keep[kTileThreads];  // kept elements of each thread
  __shared__ uint32_t s_q[kTileThreads + 1];           // first tile-local S position of each thread
  __shared__ uint64_t bar[kStages];
  __shared__ int64_t s_tile[kStages];
  __shared__ uint32_t sh_warp[2][kTileThreads / 32 + 1];
  __shared__ uint32_t sh_ex[2];
  __shared__ int s_abort;
  __shared__ uint32_t s_late;  // stages whose wait gave up (bit sg) and its parity (bit 8 + sg)

  const uint32_t T = st->prefix;
  const uint32_t need = st->rem;
  const int t = threadIdx.x;
  const int64_t n = nd.d;
  // tile prefixes from the recorded counts when available, else look-back
  const bool pre = tile_pre != nullptr && tile_counts_usable(br);
  const uint64_t policy = tc::make_policy_evict_first();

  auto fetch = [&](int sg) {  // thread 0: next ticket into stage sg
    const int64_t id = s_abort ? ntiles : int64_t(atomicAdd(ticket, 1u));
    if (id < ntiles) {
      const int64_t e0 = id * TE;
      const uint32_t bytes = uint32_t((count - e0 < TE ? count - e0 : int64_t(TE)) * int64_t(sizeof(KT)));
      tc::mbar_expect_tx(&bar[sg], bytes);
      tc::bulk_load_hint(tiles + sg * (TB / 16), W + e0, bytes, &bar[sg], policy);
    }
    s_tile[sg] = id < ntiles ? id : -1;
  };
  if (t == 0) {
    s_abort = 0;
    s_late = 0;
    for (int sg = 0; sg < kStages; ++sg) tc::mbar_init(&bar[sg], 1);
    tc::fence_mbar_init();
    // the last stage is filled at the end of the first iteration
    for (int sg = 0; sg < kStages - 1; ++sg) fetch(sg);
  }
  __syncthreads();

  // first slot of the thread: the eight threads of a quarter-warp read
  // distinct 16-byte bank groups (a thread's vectors are contiguous)
  static_assert(kTileVPT <= 8 && 8 % kTileVPT == 0, "slot rotation");
  const int r0 = (t / (8 / kTileVPT)) & (kTileVPT - 1);
  for (int it = 0;; ++it) {
    const int sg = it % kStages;
    const int64_t tile = s_tile[sg];
    if (tile < 0) break;
    // every thread observes the copy's completion on the mbarrier itself
    if (!tc::mbar_wait(&bar[sg], uint32_t(it / kStages) & 1u, err) && t == 0) {
      s_abort = 1;
      s_late |= (1u << sg) | ((uint32_t(it / kStages) & 1u) << (8 + sg));
    }
    const int64_t e0 = tile * TE;
    const int nv = int((count - e0 < TE ? count - e0 : int64_t(TE)) / EPV);
    uint4* tv = tiles + sg * (TB / 16);

    // phase 1: masks and counts of the thread's vectors, slot order r0, r0+1, ...
    uint32_t msk[kTileVPT], cnt[kTileVPT];
    uint32_t tot = 0, lo = 0;  // lo: counts of the slots before r0
#pragma unroll
    for (int kk = 0; kk < kTileVPT; ++kk) {
      const int s = (kk + r0) & (kTileVPT - 1);
      const int v = t * kTileVPT + s;
      uint32_t gm = 0, em = 0;
      if (v < nv) vec_masks<KT>(tv[v], T, gm, em);
      msk[kk] = gm | (em << 8);
      cnt[kk] = (uint32_t(__popc(gm)) << 16) | uint32_t(__popc(em));
      tot += cnt[kk];
      if (s < r0) lo += cnt[kk];
    }
    uint32_t total;
    const uint32_t ex = block_excl_scan2(tot, sh_warp, it & 1, total);
    uint32_t tg, te;  // counts of keys > T and == T in the tiles before this one
    if (pre) {
      const unsigned long long p = tile_pre[tile];
      tg = uint32_t(p >> 32);
      te = uint32_t(p);
    } else {
      if (t < 32) {
        uint32_t xg, xe;
        lookback(flags, tile, total >> 16, total & 0xFFFFu, err, xg, xe);
        if (t == 0) {
          sh_ex[0] = xg;
          sh_ex[1] = xe;
        }
      }
      __syncthreads();
      tg = sh_ex[0];
      te = sh_ex[1];
    }
    const uint32_t P0 = tg + min(need, te);  // first S position of this tile
    const uint32_t ex_gt = tg + (ex >> 16), ex_eq = te + (ex & 0xFFFFu);
    // the tile's columns: x = c0 + offset, row = row0 + x / n
    const int64_t row0 = e0 / n;
    const uint32_t c0 = uint32_t(e0 - row0 * n);

    // phase 2: kept-element masks (thread-contiguous, bit e = the thread's
    // element e in linear order), row starts, and each thread's first
    // tile-local S position
    uint64_t keep = 0;
    uint32_t run = lo;
#pragma unroll
    for (int kk = 0; kk < kTileVPT; ++kk) {
      const int s = (kk + r0) & (kTileVPT - 1);
      if (s == 0) run = 0;
      const int v = t * kTileVPT + s;
      if (v < nv) {
        const uint32_t gm = msk[kk] & 0xFFu, em = msk[kk] >> 8;
        const uint32_t cg = ex_gt + (run >> 16), ce = ex_eq + (run & 0xFFFFu);
        const uint32_t x = c0 + uint32_t(v) * EPV;
        const uint32_t q = fdiv(nd, x);
        if (x == q * uint32_t(n)) row_ptr[row0 + q] = int32_t(cg + min(need, ce));
        // ties kept in this vector: the first `allow` set bits of em
        uint32_t keq = 0;
        if (need > ce && em) {
          uint32_t allow = min(need - ce, uint32_t(__popc(em))), rest = em;
          for (; allow; --allow) {
            keq |= rest & (0u - rest);
            rest &= rest - 1u;
          }
        }
        keep |= uint64_t(gm | keq) << (s * EPV);
      }
      run += cnt[kk];
    }
    const uint32_t kept = (total >> 16) + min(need, te + (total & 0xFFFFu)) - min(need, te);
    s_keep[t] = keep;
    s_q[t] = ex_gt + min(need, ex_eq) - P0;
    if (t == 0) s_q[kTileThreads] = kept;
    __syncthreads();

    // phase 3: the tile's S entries in order, output i by thread i mod 256
    // (coalesced stores): find the owning thread u by binary search over the
    // first positions, then the (i − q_u)-th kept element of u; the element
    // is zeroed in the staged tile, which becomes the residual
    KT* te_ = reinterpret_cast<KT*>(tv);
    for (uint32_t i = t; i < kept; i += kTileThreads) {
      int u = 0;
#pragma unroll
      for (int step = kTileThreads / 2; step; step >>= 1)
        if (s_q[u + step] <= i) u += step;
      const int e = nth_set_bit64(s_keep[u], i - s_q[u]);
      const int idx = u * (kTileVPT * EPV) + e;
      const uint32_t bits = uint32_t(te_[idx]);
      const uint32_t x = c0 + uint32_t(idx);
      const uint32_t p = P0 + i;
      if (p < k) {
        col[p] = int32_t(x - fdiv(nd, x) * uint32_t(n));
        val[p] = conv_val<SB>(bits, sizeof(KT));
      }
      if (R) te_[idx] = KT(0);
    }
    if (R) tc::fence_async_smem();
    __syncthreads();
    if (t == 0) {
      if (R) {
        tc::bulk_store(R + e0, tv, uint32_t(nv) * 16u);
        tc::bulk_commit();
      }
      if (tile == ntiles - 1) row_ptr[m] = int32_t(k);
    }
    if (t == 0) {
      // the stage of the previous tile is free once its store has read it
      // (this tile's store may still be reading its own stage)
      if (R) tc::bulk_wait_read_but_one();
      fetch((it + kStages - 1) % kStages);
    }
    // no barrier here: the next tile's scan orders s_tile, and the barrier
    // before the store above ended every read of s_keep / s_q of this tile
  }
  if (t == 0) {
    tc::bulk_wait_all();
    // a copy whose wait gave up may still land: give it one more bounded wait
    for (int sg = 0; sg < kStages; ++sg)
      if ((s_late >> sg) & 1u) tc::mbar_wait(&bar[sg], (s_late >> (8 + sg)) & 1u, err);
  }
}

}  // namespace
}  // namespace hsl
