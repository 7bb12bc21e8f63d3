// Stage 1, structured: 2:4 split of W into (values, in-group indices) + residual.
//
// HASSLE-free article (aibr.jp/archives/82335), §3: N:M sparsity is the
// structured form of S that GPUs accelerate.  Rule: in each row, in every
// group of four consecutive inputs, keep the two largest |w|, ties to the
// lower in-group index, stored in ascending column order; the residual is W
// with the kept entries set to +0.0.
//
// One streaming pass: each thread reads 8 consecutive weights (two groups),
// ranks each group with six magnitude compares, writes 4 values, two index
// bytes (i0 | i1 << 2) and 8 residual words.  The value / index / residual
// arrays are flat in the same order as W, so no row bookkeeping is needed.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace hsl {
namespace {

template <typename KT> struct K24;
template <> struct K24<uint16_t> { static constexpr uint32_t kMask = 0x7FFFu, kInf = 0x7F80u; };
template <> struct K24<uint32_t> {
  static constexpr uint32_t kMask = 0x7FFFFFFFu, kInf = 0x7F800000u;
};

template <typename SB> __device__ __forceinline__ SB conv24(uint32_t bits, int src_bytes);
template <> __device__ __forceinline__ uint16_t conv24<uint16_t>(uint32_t bits, int src_bytes) {
  if (src_bytes == 2) return uint16_t(bits);
  return __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(bits)));
}
template <> __device__ __forceinline__ uint32_t conv24<uint32_t>(uint32_t bits, int src_bytes) {
  return src_bytes == 2 ? (bits << 16) : bits;
}

// Mask (4 bits) of the two kept entries of one group; sets nan on NaN keys.
template <typename KT>
__device__ __forceinline__ uint32_t keep_mask(const uint32_t (&b)[4], bool& nan) {
  uint32_t k[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    k[e] = b[e] & K24<KT>::kMask;
    nan |= k[e] > K24<KT>::kInf;
  }
  // rank[e] = entries strictly ahead of e in (|w| desc, index asc) order
  int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
  if (k[1] > k[0]) ++r0; else ++r1;
  if (k[2] > k[0]) ++r0; else ++r2;
  if (k[3] > k[0]) ++r0; else ++r3;
  if (k[2] > k[1]) ++r1; else ++r2;
  if (k[3] > k[1]) ++r1; else ++r3;
  if (k[3] > k[2]) ++r2; else ++r3;
  return uint32_t(r0 < 2) | (uint32_t(r1 < 2) << 1) | (uint32_t(r2 < 2) << 2) |
         (uint32_t(r3 < 2) << 3);
}

template <typename KT, typename SB>
__device__ __forceinline__ void do_group(const uint32_t (&b)[4], SB* val2, uint8_t* idx1,
                                         uint32_t (&rb)[4], bool& nan) {
  const uint32_t mk = keep_mask<KT>(b, nan);
  const int i0 = __ffs(mk) - 1;
  const int i1 = 31 - __clz(mk);
  val2[0] = conv24<SB>(b[i0], sizeof(KT));
  val2[1] = conv24<SB>(b[i1], sizeof(KT));
  *idx1 = uint8_t(i0 | (i1 << 2));
#pragma unroll
  for (int e = 0; e < 4; ++e) rb[e] = ((mk >> e) & 1u) ? 0u : b[e];
}

// Vector path: one thread = 8 consecutive weights = 2 groups.
template <typename KT, typename SB>
__global__ void __launch_bounds__(256) k_split_24_vec(const KT* __restrict__ W, int64_t pairs,
                                                      SB* __restrict__ val, uint8_t* __restrict__ idx,
                                                      KT* __restrict__ R, uint32_t* __restrict__ err) {
  bool nan = false;
  for (int64_t p = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; p < pairs;
       p += int64_t(gridDim.x) * blockDim.x) {
    uint32_t w[8];
    if (sizeof(KT) == 2) {
      const uint4 q = ld_stream16(W + p * 8);
      const uint32_t v4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w[2 * e] = v4[e] & 0xFFFFu;
        w[2 * e + 1] = v4[e] >> 16;
      }
    } else {
      const uint4 q0 = ld_stream16(W + p * 8), q1 = ld_stream16(W + p * 8 + 4);
      w[0] = q0.x; w[1] = q0.y; w[2] = q0.z; w[3] = q0.w;
      w[4] = q1.x; w[5] = q1.y; w[6] = q1.z; w[7] = q1.w;
    }
    SB v[4];
    uint8_t ix[2];
    uint32_t rb[8];
    {
      const uint32_t g0[4] = {w[0], w[1], w[2], w[3]};
      const uint32_t g1[4] = {w[4], w[5], w[6], w[7]};
      uint32_t r0[4], r1[4];
      do_group<KT, SB>(g0, v, &ix[0], r0, nan);
      do_group<KT, SB>(g1, v + 2, &ix[1], r1, nan);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        rb[e] = r0[e];
        rb[4 + e] = r1[e];
      }
    }
    // values: 4 per thread
    if (sizeof(SB) == 2) {
      uint2 o;
      o.x = uint32_t(v[0]) | (uint32_t(v[1]) << 16);
      o.y = uint32_t(v[2]) | (uint32_t(v[3]) << 16);
      *reinterpret_cast<uint2*>(val + p * 4) = o;
    } else {
      uint4 o;
      o.x = uint32_t(v[0]); o.y = uint32_t(v[1]); o.z = uint32_t(v[2]); o.w = uint32_t(v[3]);
      *reinterpret_cast<uint4*>(val + p * 4) = o;
    }
    *reinterpret_cast<uint16_t*>(idx + p * 2) = uint16_t(ix[0] | (ix[1] << 8));
    if (R) {
      if (sizeof(KT) == 2) {
        uint4 o;
        o.x = rb[0] | (rb[1] << 16); o.y = rb[2] | (rb[3] << 16);
        o.z = rb[4] | (rb[5] << 16); o.w = rb[6] | (rb[7] << 16);
        st_stream16(R + p * 8, o);
      } else {
        st_stream16(R + p * 8, make_uint4(rb[0], rb[1], rb[2], rb[3]));
        st_stream16(R + p * 8 + 4, make_uint4(rb[4], rb[5], rb[6], rb[7]));
      }
    }
  }
  if (__syncthreads_or(nan) && threadIdx.x == 0) set_error(err, kErrNaN);
}

// Scalar path (unaligned pointers or a group count that is odd): one group per thread.
template <typename KT, typename SB>
__global__ void __launch_bounds__(256) k_split_24_scalar(const KT* __restrict__ W, int64_t groups,
                                                         SB* __restrict__ val,
                                                         uint8_t* __restrict__ idx,
                                                         KT* __restrict__ R,
                                                         uint32_t* __restrict__ err) {
  bool nan = false;
  for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += int64_t(gridDim.x) * blockDim.x) {
    const uint32_t b[4] = {uint32_t(W[4 * g]), uint32_t(W[4 * g + 1]), uint32_t(W[4 * g + 2]),
                           uint32_t(W[4 * g + 3])};
    uint32_t rb[4];
    do_group<KT, SB>(b, val + 2 * g, idx + g, rb, nan);
    if (R)
#pragma unroll
      for (int e = 0; e < 4; ++e) R[4 * g + e] = KT(rb[e]);
  }
  if (__syncthreads_or(nan) && threadIdx.x == 0) set_error(err, kErrNaN);
}

template <typename KT, typename SB>
hsl_status run24(Handle& h, const KT* W, KT* R, cudaStream_t s) {
  const int64_t groups = h.m * h.n / 4;
  SB* val = static_cast<SB*>(h.nm_val.p);
  uint8_t* idx = static_cast<uint8_t*>(h.nm_idx.p);
  uint32_t* err = static_cast<uint32_t*>(h.err.p);
  const bool vec_ok = groups % 2 == 0 && reinterpret_cast<uintptr_t>(W) % 16 == 0 &&
                      (R == nullptr || reinterpret_cast<uintptr_t>(R) % 16 == 0);
  const int threads = 256;
  if (vec_ok) {
    const int64_t pairs = groups / 2;
    const int64_t grid = std::min<int64_t>((pairs + threads - 1) / threads, int64_t(h.num_sms) * 16);
    k_split_24_vec<KT, SB><<<unsigned(std::max<int64_t>(grid, 1)), threads, 0, s>>>(W, pairs, val,
                                                                                    idx, R, err);
  } else {
    const int64_t grid = std::min<int64_t>((groups + threads - 1) / threads, int64_t(h.num_sms) * 16);
    k_split_24_scalar<KT, SB><<<unsigned(std::max<int64_t>(grid, 1)), threads, 0, s>>>(
        W, groups, val, idx, R, err);
  }
  note_launch();
  return cuda_fail(cudaGetLastError(), "2:4 split launch");
}

}  // namespace

hsl_status split_24_run(Handle& h, const void* W, hsl_dtype wdt, void* R, cudaStream_t s) {
  const size_t half = size_t(h.m) * size_t(h.n / 2);
  if (hsl_status e = ensure(h.nm_val, half * dtype_bytes(h.dtype), "2:4 values")) return e;
  if (hsl_status e = ensure(h.nm_idx, size_t(h.m) * size_t(h.n / 4), "2:4 indices")) return e;
  if (wdt == HSL_BF16) {
    if (h.dtype == HSL_BF16)
      return run24<uint16_t, uint16_t>(h, static_cast<const uint16_t*>(W), static_cast<uint16_t*>(R), s);
    return run24<uint16_t, uint32_t>(h, static_cast<const uint16_t*>(W), static_cast<uint16_t*>(R), s);
  }
  if (h.dtype == HSL_BF16)
    return run24<uint32_t, uint16_t>(h, static_cast<const uint32_t*>(W), static_cast<uint32_t*>(R), s);
  return run24<uint32_t, uint32_t>(h, static_cast<const uint32_t*>(W), static_cast<uint32_t*>(R), s);
}

}  // namespace hsl
