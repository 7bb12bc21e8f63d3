// Small-batch (2..64 tokens) 2:4 apply on the sparse tensor cores, K split
// across every SM.
//
// "Hierarchical Sparse + Low-Rank Compression of LLMs", §Implementation and
// operational patterns: y = S x + U (Vᵀ x).  At a handful of tokens the cost is
// streaming S once from HBM (SqueezeLLM article, §1), but the per-token work
// (16 tokens × 2 products per kept weight) is too much for the CUDA cores to
// keep up with the memory system, so the S·Xᵀ part runs on the 2:4 sparse MMA
// as in the prefill kernel.  What differs is how the work is cut: a layer has
// only m/128 row tiles (86 for 11008 rows), far fewer than the SMs × CTAs per
// SM, so the (row tile, 64-column K-block) units of the whole layer are dealt
// out in equal contiguous ranges to a persistent grid of one CTA per SM.
//
//   k_splitk_z   z = Vᵀ x for the T tokens in fp32 (a warp per (row of Vt,
//                8 tokens), fixed shuffle-tree sums); triggers the dependent
//                launch at its start.
//   k_apply_24_splitk<TP>  a unit is a 128-row tile × two 64-column K-blocks:
//                one 16 KB TMA of the 128×64 compressed values (128-byte
//                swizzle; a copy instruction costs a near-fixed time, so
//                16 KB per instruction streams about twice as fast as 8 KB),
//                the two X blocks [TP tokens × 64] in one 3-D box (128-byte
//                swizzle, tokens past T zero-filled) and 2 KB of TMEM-ordered metadata by
//                bulk copy, written into TMEM by tcgen05.st; four
//                tcgen05.mma.sp of K = 32 into a 128×TP fp32 accumulator in
//                TMEM.  A CTA's range covers the end
//                of one tile and the start of the next (or a whole tile), so it
//                keeps two accumulators and hands each finished tile segment to
//                its epilogue warps.
//   Combining a tile's segments: a segment that is a whole tile is finished
//   in place (+ U·z, rounded to bf16).  Otherwise each segment's CTA stores
//   its fp32 partial in its own slot (tile + CTA index: unique), counts itself
//   in on the tile's counter, and the CTA that arrives last adds the slots in
//   CTA order, then U·z, and rounds — the same order whichever CTA is last, so
//   the result is deterministic.  That CTA resets the counter for the next
//   call.  Nobody waits on anybody: no spin on another CTA.
//
// Warp roles (384 threads): lane 0 of warp 0 issues the S copies, of warp 10
// the X copies and of warp 11 the metadata copy (three issuers, so their copy
// instructions overlap); warps 2-5 write each unit's metadata into TMEM
// (tcgen05.st) once it has landed; the S and X copies and those 128 threads
// complete the unit's one `full` barrier, on which lane 0 of warp 1 (which owns
// TMEM) waits before the unit's MMAs; warps 6-9 run the epilogues (TMEM lane
// quarter = warp % 4).  Every wait is
// bounded; a wait that gives up sets the error word, and the CTA still drains
// its copies, takes part in the tile counters and frees TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hsl {
namespace {

constexpr int SK_THREADS = 384;    // 12 warps (roles below)
constexpr int SK_A = 128 * 128;     // compressed values of a unit: 128 rows × 128 bytes (2 K-blocks)
constexpr int SK_M = 2 * 128 * 8;   // TMEM-ordered metadata of the unit's 2 K-blocks (compact)
constexpr uint32_t SK_TMEM_COLS = 256;
// accumulator b at TMEM column 64·b
__host__ __device__ constexpr uint32_t sk_acc_col(int b) { return 64u * uint32_t(b); }

// stages per token padding: the ring and z (TP rows × up to 256 fp32, staged
// once for the U·z sums of the tiles the CTA finishes) share 200 KB of shared
// memory; at most 8 stages (their metadata slots fill TMEM columns [128, 256))
__host__ __device__ constexpr int sk_stage_bytes(int tp) { return SK_A + 2 * tp * 128 + SK_M; }
__host__ __device__ constexpr int sk_zbytes(int tp) { return tp * 256 * 4; }
__host__ __device__ constexpr int sk_stages(int tp) {
  return (200 * 1024 - sk_zbytes(tp)) / sk_stage_bytes(tp) < 8
             ? (200 * 1024 - sk_zbytes(tp)) / sk_stage_bytes(tp)
             : 8;
}
static_assert(sk_stages(16) == 8 && sk_stages(64) >= 3, "stage counts");
__host__ __device__ constexpr int sk_smem(int tp) {
  return sk_stages(tp) * sk_stage_bytes(tp) + sk_zbytes(tp) + 1024 + 256;
}
// metadata slot of (stage, MMA i): 4-column aligned, after both accumulators
__device__ __forceinline__ uint32_t sk_meta_col(int s, int i) { return 128u + 16u * s + 4u * i; }

struct SkMaps {
  CUtensorMap sv;  // S values [m][n/2]  box {64, 128} SW128 (two K-blocks of 64 columns)
  CUtensorMap x;   // X [T][n] as [n/64][T][64], box {64, TP, 2} SW128 (both X blocks of a unit)
};

struct SkArgs {
  const uint2* meta;        // TMEM-ordered 2:4 metadata [tiles][nkb][128]
  const __nv_bfloat16* U;   // [m][r_pad]
  const float* z;           // [T][r_pad]
  float* part;              // partial tiles [(tiles + grid)][TP][128]
  unsigned* cnt;            // [tiles]
  __nv_bfloat16* Y;         // [T][m]
  uint32_t* err;
  int m, n, T, r, r_pad, nkb, tiles;  // nkb: units per tile (pairs of 64-column K-blocks)
  long long units;          // tiles · nkb
};

// CTA c of `grid` owns units [c·units/grid, (c+1)·units/grid)
__device__ __forceinline__ long long unit_begin(long long c, long long units, int grid) {
  return c * units / grid;
}
// the CTA whose range holds unit u
__device__ __forceinline__ int cta_of(long long u, long long units, int grid) {
  return int(((u + 1) * grid - 1) / units);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, uint32_t* err,
                                              volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (tc::mbar_wait(bar, parity, err)) return true;
  *abort_flag = 1;
  return false;
}

// 16 consecutive fp32 TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// named barrier over the four epilogue warps
__device__ __forceinline__ void epi_sync() { asm volatile("barrier.sync 1, 128;" ::: "memory"); }

// ---- z = Vᵀ x ------------------------------------------------------------------
// Work items (row c of Vt, 8 tokens) are cut into pieces of 256 columns, a warp
// per piece (16-byte loads of the row and of the 8 tokens, fixed shuffle
// trees), so thousands of warps share the V stream.  Each piece's 8 sums go to
// its own slot; the warp that finishes an item last (a counter per item)
// adds the item's pieces in piece order and writes z, then resets the counter:
// the result does not depend on timing, and no warp waits for another.
constexpr int kSkZThreads = 256;
constexpr int kSkZPiece = 256;  // columns per piece
__global__ void __launch_bounds__(kSkZThreads) k_splitk_z(const __nv_bfloat16* __restrict__ Vt,
                                                          const __nv_bfloat16* __restrict__ X,
                                                          float* __restrict__ z, int n, int T,
                                                          int r, int r_pad, float* __restrict__ zpart,
                                                          unsigned* __restrict__ zcnt) {
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int tb_count = (T + 7) / 8;
  const int Q = (n + kSkZPiece - 1) / kSkZPiece;
  const long long items = (long long)r * tb_count;
  const long long total = items * Q;
  const long long nw = (long long)gridDim.x * (kSkZThreads / 32);
  for (long long it = ((long long)blockIdx.x * kSkZThreads + threadIdx.x) >> 5; it < total; it += nw) {
    const long long item = it / Q;
    const int q = int(it - item * Q);
    const int c = int(item / tb_count), tb = int(item % tb_count);
    const int t0 = tb * 8;
    const int j = q * kSkZPiece + lane * 8;
    float acc[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[b] = 0.f;
    if (j < n) {
      const uint4 v = ld_stream16(Vt + (long long)c * n + j);
      const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
      uint4 xq[8];
#pragma unroll
      for (int b = 0; b < 8; ++b)
        if (t0 + b < T) xq[b] = *reinterpret_cast<const uint4*>(X + (long long)(t0 + b) * n + j);
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        if (t0 + b < T) {
          const uint32_t xw[4] = {xq[b].x, xq[b].y, xq[b].z, xq[b].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[b] = fmaf(bf_lo(vw[e]), bf_lo(xw[e]), acc[b]);
            acc[b] = fmaf(bf_hi(vw[e]), bf_hi(xw[e]), acc[b]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < 8; ++b)
#pragma unroll
      for (int o = 16; o; o >>= 1) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], o);
    float* slot = zpart + (item * Q + q) * 8;
    if (lane < 8) {
      float mine = acc[0];
#pragma unroll
      for (int b = 1; b < 8; ++b)
        if (lane == b) mine = acc[b];
      slot[lane] = mine;
    }
    __threadfence();
    __syncwarp();
    unsigned last = 0;
    if (lane == 0) last = atomicAdd(&zcnt[item], 1u) == unsigned(Q - 1);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __threadfence();
      if (lane < 8 && t0 + lane < T) {
        float zv = 0.f;
        for (int qq = 0; qq < Q; ++qq) zv += __ldcg(zpart + (item * Q + qq) * 8 + lane);
        z[(long long)(t0 + lane) * r_pad + c] = zv;
      }
      if (lane == 0) zcnt[item] = 0u;  // ready for the next call
    }
  }
}

// ---- the split-K kernel ------------------------------------------------------------
template <int TP>
__global__ void __launch_bounds__(SK_THREADS, 1)
    k_apply_24_splitk(const __grid_constant__ SkMaps maps, const SkArgs a) {
  constexpr int ST = sk_stages(TP);
  constexpr int STAGE = sk_stage_bytes(TP);
  constexpr int B_BYTES = TP * 128;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* zs = reinterpret_cast<float*>(smem + ST * STAGE);  // [TP][r_pad], staged once
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * STAGE + sk_zbytes(TP));
  uint64_t* mload = full + ST;  // the unit's metadata has landed
  uint64_t* empty = mload + ST;
  uint64_t* accfull = empty + ST;   // [2]
  uint64_t* accempty = accfull + 2; // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 2);
  __shared__ int abort_flag;
  __shared__ int last_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grid = int(gridDim.x);
  const long long u0 = unit_begin(blockIdx.x, a.units, grid);
  const long long u1 = unit_begin((long long)blockIdx.x + 1, a.units, grid);
  const int nkb = a.nkb;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      // the S and X issuers, and the 128 threads that put the unit's metadata
      // into TMEM: the MMA thread waits on this one barrier per unit (a wait on a
      // completed phase costs that thread a few hundred cycles after MMA issue)
      tc::mbar_init(&full[s], 2 + 128);
      tc::mbar_init(&mload[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&accfull[b], 1);
      tc::mbar_init(&accempty[b], 128);
    }
    tc::fence_mbar_init();
    tc::prefetch_tmap(&maps.sv);
    tc::prefetch_tmap(&maps.x);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, SK_TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abrt = &abort_flag;

  if (warp == 0 || warp >= 10) {
    // warp 0: the unit's S values; warp 10: its two X blocks; warp 11: its metadata
    if (lane == 0) {
      const uint64_t keep = tc::make_policy_evict_last();
      const uint64_t stream = tc::make_policy_evict_first();
      // (tile, K-block pair) of the unit advanced incrementally: a single
      // thread's 64-bit division would cost hundreds of cycles per unit
      int tile = int(u0 / nkb), kp = int(u0 % nkb);
      const int nu = int(u1 - u0);
      int k = 0, s = 0;
      uint32_t ph = 0;
      for (; k < nu; ++k) {
        if (!wait_or_abort(&empty[s], ph ^ 1, a.err, abrt)) break;
        unsigned char* st = smem + s * STAGE;
        if (warp == 0) {
          tc::mbar_expect_tx(&full[s], SK_A);
          tc::tma_load_2d_hint(st, &maps.sv, kp * 64, tile * 128, &full[s], stream);
        } else if (warp == 10) {
          // one copy for both X blocks: a copy instruction holds its issuing
          // thread for a near-fixed time whatever its size
          tc::mbar_expect_tx(&full[s], 2 * B_BYTES);
          tc::tma_load_3d_hint(st + SK_A, &maps.x, 0, 0, kp * 2, &full[s], keep);
        } else {
          // the metadata of K-blocks 2·kp and 2·kp + 1 lie next to each other
          tc::mbar_expect_tx(&mload[s], SK_M);
          tc::bulk_load(st + SK_A + 2 * B_BYTES, a.meta + ((long long)tile * nkb + kp) * 256, SK_M,
                        &mload[s]);
        }
        if (++kp == nkb) { kp = 0; ++tile; }
        if (++s == ST) { s = 0; ph ^= 1u; }
      }
      // drain: the stages of the last (up to ST) units this thread issued have landed
      // (the S and X copies complete the same phases of `full`; the metadata
      // completes on `mload`)
      uint64_t* landed = warp == 11 ? mload : full;
      for (int j = k > ST ? k - ST : 0; j < k; ++j) tc::mbar_wait(&landed[j % ST], (j / ST) & 1, a.err);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_sp = tc::idesc_bf16(128, TP) | (1u << 2);
      int seg = -1;
      const int nu = int(u1 - u0);
      int kb = int(u0 % nkb), s = 0;
      uint32_t ph = 0;
      for (int k = 0; k < nu; ++k, kb = (kb + 1 == nkb ? 0 : kb + 1), s = (s + 1 == ST ? 0 : s + 1),
               ph ^= (s == 0 ? 1u : 0u)) {
        const bool first = k == 0 || kb == 0;
        const bool last = k + 1 == nu || kb == nkb - 1;
        if (first) {
          ++seg;
          // the accumulator of two segments back must have been read out
          if (seg >= 2 && !wait_or_abort(&accempty[seg & 1], ((seg - 2) >> 1) & 1, a.err, abrt))
            break;
        }
        if (!wait_or_abort(&full[s], ph, a.err, abrt)) break;
        tc::tc_fence_after();
        const unsigned char* st = smem + s * STAGE;
        const uint64_t ad = tc::desc_sw128(st);
        const uint32_t d = tmem + sk_acc_col(seg & 1);
        // MMA i: K-block i / 2 (its X block), 32 logical columns (i % 2) of it;
        // the values advance 32 bytes per MMA within their 128-byte rows
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint64_t bd = tc::desc_sw128(st + SK_A + (i >> 1) * B_BYTES);
          tc::mma_bf16_sp(d, tc::desc_advance(ad, 32 * i), tc::desc_advance(bd, 64 * (i & 1)),
                          tmem + sk_meta_col(s, i), idesc_sp, (!first || i > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
        if (last) tc::mma_commit(&accfull[seg & 1]);
      }
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp < 6) {
    // metadata of each unit into its TMEM slots (one 32-bit column per lane and
    // MMA), then an arrival on the unit's `full` barrier, so the MMA thread
    // waits on that one barrier.  A warp reaches TMEM lanes 32·(warp % 4) onwards.
    const int L = ((warp & 3) << 5) | lane;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    int s = 0;
    uint32_t ph = 0;
    for (long long u = u0; u < u1; ++u) {
      // the unit's metadata has landed, so the MMAs of its stage's previous use
      // (the last readers of these TMEM slots) are done
      if (!wait_or_abort(&mload[s], ph, a.err, abrt)) break;
      const unsigned char* st = smem + s * STAGE;
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        const uint2 w = *reinterpret_cast<const uint2*>(st + SK_A + 2 * B_BYTES + kb * 1024 + L * 8);
        tc::tmem_st1(tmem + lane_base + sk_meta_col(s, 2 * kb), w.x);
        tc::tmem_st1(tmem + lane_base + sk_meta_col(s, 2 * kb + 1), w.y);
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(&full[s]);
      if (++s == ST) { s = 0; ph ^= 1u; }
    }
  } else {
    // epilogue: one tile segment at a time; TMEM lane = row of the tile
    const int q = warp & 3;
    const int L = (q << 5) | lane;
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    const int tid = threadIdx.x - 192;  // 0..127 over the epilogue warps
    bool z_ready = false;
    int seg = 0;
    for (long long u = u0; u < u1; ++seg) {
      const int tile = int(u / nkb);
      const long long tile_u0 = (long long)tile * nkb, tile_u1 = tile_u0 + nkb;
      const long long seg_end = tile_u1 < u1 ? tile_u1 : u1;
      const int c_first = cta_of(tile_u0, a.units, grid);
      const int c_last = cta_of(tile_u1 - 1, a.units, grid);
      const int nseg = c_last - c_first + 1;
      // this row's U into L2 while the segment's MMAs run (the CTA that finishes
      // the tile reads it after the partial sums; from DRAM each of its loads
      // would cost a full memory latency)
      if (a.r > 0 && tile * 128 + L < a.m) {
        const char* up = reinterpret_cast<const char*>(a.U + (long long)(tile * 128 + L) * a.r_pad);
        for (int b = 0; b < a.r_pad * 2; b += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(up + b));
      }
      float v[TP];
      const bool ok = wait_or_abort(&accfull[seg & 1], (seg >> 1) & 1, a.err, abrt);
      if (ok) {
        tc::tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < TP; c0 += 16)
          tmem_ld16(tmem + lane_base + sk_acc_col(seg & 1) + c0, v + c0);
      } else {
#pragma unroll
        for (int t = 0; t < TP; ++t) v[t] = 0.f;
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&accempty[seg & 1]);
      const int i = tile * 128 + L;
      bool finish = nseg == 1;
      if (!finish) {
        // this CTA's partial into its own slot, then count in on the tile
        float* slot = a.part + ((long long)tile + blockIdx.x) * TP * 128;
#pragma unroll
        for (int t = 0; t < TP; ++t) slot[t * 128 + L] = v[t];
        __threadfence();
        epi_sync();
        if (tid == 0) {
          const unsigned old = atomicAdd(&a.cnt[tile], 1u);
          last_flag = old == unsigned(nseg - 1);
        }
        epi_sync();
        finish = last_flag != 0;
        if (finish) {
          __threadfence();
          // the slots of the tile's CTAs, added in CTA order
#pragma unroll
          for (int t = 0; t < TP; ++t) v[t] = 0.f;
          for (int j = 0; j < nseg; ++j) {
            const float* sl = a.part + ((long long)tile + c_first + j) * TP * 128;
#pragma unroll
            for (int t = 0; t < TP; ++t) v[t] += __ldcg(sl + t * 128 + L);
          }
          if (tid == 0) a.cnt[tile] = 0u;  // ready for the next call
        }
      }
      if (finish && a.r > 0 && !z_ready) {
        // z into shared memory, once: the sums below read it for every row
        pdl_wait();  // z is written by the preceding kernel
        for (int e = tid; e < TP * a.r_pad / 4; e += 128)
          reinterpret_cast<float4*>(zs)[e] = __ldcg(reinterpret_cast<const float4*>(a.z) + e);
        epi_sync();
        z_ready = true;
      }
      if (finish && i < a.m) {
        if (a.r > 0) {
          // + U[i,:]·z[t,:], added to the tile's sum in factor-column order (fp32).
          // Two 16-byte pieces of the U row are loaded before either is used; z
          // has TP rows (rows past T hold whatever the last call left; their
          // sums are never stored), so its reads need no guard.
          const __nv_bfloat16* urow = a.U + (long long)i * a.r_pad;
          for (int c0 = 0; c0 < a.r_pad; c0 += 16) {
            uint4 uq[2];
#pragma unroll
            for (int j = 0; j < 2; ++j)
              uq[j] = c0 + 8 * j < a.r_pad ? *reinterpret_cast<const uint4*>(urow + c0 + 8 * j)
                                          : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int c = c0 + 8 * j;
              if (c >= a.r_pad) break;
              const float uf[8] = {bf_lo(uq[j].x), bf_hi(uq[j].x), bf_lo(uq[j].y), bf_hi(uq[j].y),
                                   bf_lo(uq[j].z), bf_hi(uq[j].z), bf_lo(uq[j].w), bf_hi(uq[j].w)};
#pragma unroll
              for (int t = 0; t < TP; ++t) {
                const float4 z0 = *reinterpret_cast<const float4*>(zs + t * a.r_pad + c);
                const float4 z1 = *reinterpret_cast<const float4*>(zs + t * a.r_pad + c + 4);
                float acc = v[t];
                acc = fmaf(uf[0], z0.x, acc);
                acc = fmaf(uf[1], z0.y, acc);
                acc = fmaf(uf[2], z0.z, acc);
                acc = fmaf(uf[3], z0.w, acc);
                acc = fmaf(uf[4], z1.x, acc);
                acc = fmaf(uf[5], z1.y, acc);
                acc = fmaf(uf[6], z1.z, acc);
                acc = fmaf(uf[7], z1.w, acc);
                v[t] = acc;
              }
            }
          }
        }
#pragma unroll
        for (int t = 0; t < TP; ++t)
          if (t < a.T) __stcs(a.Y + (long long)t * a.m + i, __float2bfloat16_rn(v[t]));
      }
      u = seg_end;
    }
  }
  tc::tc_fence_before();
  tc::cta_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, SK_TMEM_COLS);
  }
}

template <int TP>
hsl_status launch_tp(Handle& h, const void* X, void* Y, int64_t T, cudaStream_t s) {
  const int64_t m = h.m, n = h.n;
  const int nkb = int(n / 128);  // units per tile: pairs of 64-column K-blocks
  const int tiles = int((m + 127) / 128);
  const long long units = (long long)tiles * nkb;
  auto kern = k_apply_24_splitk<TP>;
  const int smem = sk_smem(TP);
  if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(kern), smem))
    return cuda_fail(e, "split-K smem attribute");
  // one CTA per SM (its stage ring takes most of the shared memory)
  const int grid = int(std::min<long long>(h.num_sms, units));

  // workspace: partial slots (tile + CTA index), tile counters (zero at rest), z
  const size_t part_bytes = size_t(tiles + grid) * TP * 128 * 4;
  if (hsl_status e = ensure(h.sk_part, part_bytes, "split-K partial tiles")) return e;
  if (h.sk_cnt.bytes < size_t(tiles) * 4 || !h.sk_cnt.p) {
    if (hsl_status e = ensure(h.sk_cnt, size_t(tiles) * 4, "split-K tile counters")) return e;
    if (cudaError_t e = cudaMemsetAsync(h.sk_cnt.p, 0, h.sk_cnt.bytes, s))
      return cuda_fail(e, "split-K counter init");
  }
  const int r_pad = int(h.r_pad);
  const long long zitems = (long long)h.r * ((T + 7) / 8);
  const int zQ = int((n + kSkZPiece - 1) / kSkZPiece);
  if (h.r > 0) {
    // per-item counters first (a fixed place, zero at rest: kept across calls),
    // then z, then the pieces' partial sums
    const size_t cb = size_t(round_up(int64_t(h.r) * 8 * 4, 256));  // items for T up to 64
    const size_t zb = size_t(round_up(int64_t(TP) * r_pad * 4, 256));  // TP rows: the epilogue reads all
    const size_t pb = size_t(zitems) * zQ * 8 * 4;
    const bool fresh = !h.sk_z.p || h.sk_z.bytes < cb + zb + pb;
    if (hsl_status e = ensure(h.sk_z, cb + zb + pb, "split-K z")) return e;
    if (fresh) {
      if (cudaError_t e = cudaMemsetAsync(h.sk_z.p, 0, cb, s)) return cuda_fail(e, "split-K z counters");
    }
    h.sk_zcnt_off = 0;
    h.sk_zout_off = cb;
    h.sk_zpart_off = cb + zb;
  }

  SkMaps maps;
  memset(&maps, 0, sizeof(maps));
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_tmap_2d(&maps.sv, BF, 2, h.nm_val.p, m, n / 2, n / 2, 64, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_kblocks(&maps.x, X, T, n, TP, 2)) {
    set_message("tensor map encoding failed");
    return HSL_ERR_CUDA;
  }
  SkArgs a;
  a.meta = static_cast<const uint2*>(h.pmeta_tc.p);
  a.U = static_cast<const __nv_bfloat16*>(h.U.p);
  a.z = reinterpret_cast<const float*>(static_cast<const char*>(h.sk_z.p) + h.sk_zout_off);
  a.part = static_cast<float*>(h.sk_part.p);
  a.cnt = static_cast<unsigned*>(h.sk_cnt.p);
  a.Y = static_cast<__nv_bfloat16*>(Y);
  a.err = static_cast<uint32_t*>(h.err.p);
  a.m = int(m);
  a.n = int(n);
  a.T = int(T);
  a.r = h.r;
  a.r_pad = r_pad;
  a.nkb = nkb;
  a.tiles = tiles;
  a.units = units;

  if (h.r > 0) {
    const long long warps = zitems * zQ;
    const long long zgrid = std::min<long long>((warps * 32 + kSkZThreads - 1) / kSkZThreads,
                                                (long long)h.num_sms * 8);
    char* zb = static_cast<char*>(h.sk_z.p);
    k_splitk_z<<<unsigned(zgrid), kSkZThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(h.Vt.p), static_cast<const __nv_bfloat16*>(X),
        reinterpret_cast<float*>(zb + h.sk_zout_off), int(n), int(T), h.r, r_pad,
        reinterpret_cast<float*>(zb + h.sk_zpart_off), reinterpret_cast<unsigned*>(zb + h.sk_zcnt_off));
    note_launch();
    if (hsl_status e = cuda_fail(cudaGetLastError(), "split-K z launch")) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(SK_THREADS);
  cfg.dynamicSmemBytes = size_t(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = h.r > 0 ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cuda_fail(cudaLaunchKernelEx(&cfg, kern, maps, a), "split-K apply launch");
}

}  // namespace

bool splitk_supported(const Handle& h, const void* X, int64_t T) {
  return h.fmt == HSL_FMT_NM24 && h.dtype == HSL_BF16 && h.n % 128 == 0 && h.pmeta_tc.p &&
         T >= kSplitKMinBatch && T <= kSplitKMaxBatch && h.r <= 256 &&
         (reinterpret_cast<uintptr_t>(X) % 16) == 0 && tmap_available();
}

hsl_status apply_splitk_run(Handle& h, const void* X, void* Y, int64_t T, cudaStream_t s) {
  if (T <= 16) return launch_tp<16>(h, X, Y, T, s);
  if (T <= 32) return launch_tp<32>(h, X, Y, T, s);
  if (T <= 48) return launch_tp<48>(h, X, Y, T, s);
  return launch_tp<64>(h, X, Y, T, s);
}

}  // namespace hsl
