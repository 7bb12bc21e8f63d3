// Large-batch (prefill) apply on tcgen05 tensor cores, 2:4 S, bf16.
//
// "Hierarchical Sparse + Low-Rank Compression of LLMs", §Implementation and
// operational patterns: y = S x + U (Vᵀ x).  With many tokens both products
// are dense contractions, so they run on the 5th-generation tensor cores:
//
//   k_prefill_z    Z = X·V  ([T][r16] bf16).  M = 128 tokens per CTA, N = r16,
//                  K = n, operands by TMA (128-byte swizzle), fp32 accumulator
//                  in TMEM, bf16 epilogue.  Triggers the dependent launch at
//                  its start.
//   k_prefill_24sp the default: Yᵀ tile [256 rows of W × 224 tokens], two
//                  128-row TMEM accumulators sharing every X tile; the 2:4
//                  part runs on the sparse MMA (tcgen05.mma.sp, compressed
//                  values straight from TMA, metadata in TMEM), the low-rank
//                  part on dense MMAs (A = U, B = Z) into the same
//                  accumulators.  See the comment above the kernel.
//   k_prefill_24   the same product with each 2:4 tile expanded to dense bf16
//                  in shared memory (twice the S work on the dense MMA), one
//                  128×256 accumulator.  Kept as a cross-check of the sparse
//                  kernel (selected by HSL_PREFILL_EXPAND=1).
//   In both, the producer waits for the Z kernel (griddepcontrol.wait) only
//   before the first Z tile, so the S·Xᵀ part overlaps it; the epilogue reads
//   TMEM (tcgen05.ld), rounds to bf16 and stores Y[t][i] with streaming stores.
//
// Why 256×224 tiles: with a 2:4 sparse MMA the tensor work per byte of X halves,
// so the X traffic per flop decides whether L2 can feed the MMAs; sharing each
// X tile across 256 rows of W lowers the bytes per flop about 1.6× against a
// 128×256 tile.  And the MMA thread's loop costs about the same per K-block
// whatever N, so the widest tile TMEM allows pays: 2×224 accumulator columns
// plus the 4-column-aligned metadata slots of four stages (the sparse MMA
// requires that alignment); 1.15 ms against 1.25 ms with 192 tokens and five
// stages on the 70B layer at 4096 tokens.
//
// Warp roles: warp 0 lane 0 issues TMA; warp 1 owns TMEM and lane 0 issues
// MMAs; warps 2-5 move metadata (or expand S) and run the epilogue.  The
// sparse kernel adds warps 6 and 7, which issue the X and metadata copies.  All waits are bounded (kSpinLimit polls); a wait that gives up sets
// the error word and the CTA drains its copies, frees TMEM and exits.
#include <cuda.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hsl {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;             // 16 KB dense A tile
constexpr int B_BYTES = BN * BK * 2;             // 32 KB B tile
constexpr int SV_BYTES = BM * (BK / 2) * 2;      // 8 KB compressed values
constexpr int SI_BYTES = BM * (BK / 4);          // 2 KB index bytes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SV_BYTES + SI_BYTES;
constexpr int PREFILL_SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

// Z kernel: A = X tile [128 × 64], B = Vt tile [r16 × 64]
constexpr int ZSTAGES = 4;
constexpr int ZA_BYTES = 128 * BK * 2;
constexpr int ZB_MAX = 256 * BK * 2;
constexpr int Z_SMEM = ZSTAGES * (ZA_BYTES + ZB_MAX) + 1024 + 256;

struct PrefillMaps {
  CUtensorMap x;    // X  [T][n]      box {64, 256}  (main) / {64, 128} (z)
  CUtensorMap xz;   // X  [T][n]      box {64, 128}
  CUtensorMap sv;   // S values [m][n/2] box {32, 128}
  CUtensorMap si;   // S index bytes [m][n/4] box {16, 128}
  CUtensorMap u;    // U  [m][r_pad]  box {64, 128}
  CUtensorMap z;    // Z  [T][r16]    box {64, 256}
  CUtensorMap vt;   // Vt [r16][n]    box {64, r16}
};

// ---- 2:4 expansion: byte selectors for __byte_perm(vals, 0, sel) ----------
// vals = v0 | v1 << 16 (the two kept values of a group), nibble = i0 | i1 << 2.
// Returns (sel_lo | sel_hi << 16): the dense elements {e0,e1} and {e2,e3}.
__host__ __device__ constexpr uint32_t expand_sel(uint32_t nib) {
  uint32_t i0 = nib & 3u, i1 = nib >> 2;
  uint32_t s = 0;
  for (uint32_t k = 0; k < 4; ++k) {
    uint32_t lo_byte = (k == i0) ? 0u : (k == i1) ? 2u : 4u;  // byte 4+ of the second operand = 0
    uint32_t two = lo_byte | ((lo_byte + 1u) << 4);
    s |= two << (8 * k);
  }
  return s;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, uint32_t* err,
                                              volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (tc::mbar_wait(bar, parity, err)) return true;
  *abort_flag = 1;
  return false;
}

__global__ void __launch_bounds__(192, 1)
    k_prefill_24(const __grid_constant__ PrefillMaps maps, __nv_bfloat16* __restrict__ Y, int m,
                 int n, int T, int r16, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;
  unsigned char* sB = sA + STAGES * A_BYTES;
  unsigned char* sV = sB + STAGES * B_BYTES;
  unsigned char* sI = sV + STAGES * SV_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sI + STAGES * SI_BYTES);
  uint64_t* expd = full + STAGES;
  uint64_t* empty = expd + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  __shared__ uint32_t sel_tab[16];
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntn = (T + BN - 1) / BN;
  const int mt = blockIdx.x / ntn, nt = blockIdx.x % ntn;
  const int i0 = mt * BM, t0 = nt * BN;
  const int nkS = (n + BK - 1) / BK;
  const int nkL = (r16 + BK - 1) / BK;
  const int nk = nkS + nkL;

  if (threadIdx.x < 16) sel_tab[threadIdx.x] = expand_sel(threadIdx.x);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&expd[s], 128);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accf, 1);
    tc::fence_mbar_init();
    tc::prefetch_tmap(&maps.x);
    tc::prefetch_tmap(&maps.sv);
    tc::prefetch_tmap(&maps.si);
    if (r16 > 0) {
      tc::prefetch_tmap(&maps.u);
      tc::prefetch_tmap(&maps.z);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, BN);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abrt = &abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      // X and Z tiles are re-read by every 128-row tile: keep them in L2;
      // S and U are read by few CTAs in a row: let them leave L2 first.
      const uint64_t keep = tc::make_policy_evict_last();
      const uint64_t stream = tc::make_policy_evict_first();
      int issued[STAGES] = {0, 0, 0};
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!wait_or_abort(&empty[s], ph ^ 1, err, abrt)) break;
        if (kb < nkS) {
          tc::mbar_expect_tx(&full[s], B_BYTES + SV_BYTES + SI_BYTES);
          tc::tma_load_2d_hint(sB + s * B_BYTES, &maps.x, kb * BK, t0, &full[s], keep);
          tc::tma_load_2d_hint(sV + s * SV_BYTES, &maps.sv, kb * (BK / 2), i0, &full[s], stream);
          tc::tma_load_2d_hint(sI + s * SI_BYTES, &maps.si, kb * (BK / 4), i0, &full[s], stream);
        } else {
          if (kb == nkS) pdl_wait();  // Z is written by the preceding kernel
          const int kl = kb - nkS;
          tc::mbar_expect_tx(&full[s], A_BYTES + B_BYTES);
          tc::tma_load_2d_hint(sA + s * A_BYTES, &maps.u, kl * BK, i0, &full[s], stream);
          tc::tma_load_2d_hint(sB + s * B_BYTES, &maps.z, kl * BK, t0, &full[s], keep);
        }
        ++issued[s];
      }
      // drain: every copy this thread started has landed before the CTA exits
      for (int s = 0; s < STAGES; ++s)
        if (issued[s]) tc::mbar_wait(&full[s], (issued[s] - 1) & 1, err);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(BM, BN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        const bool ok = kb < nkS ? wait_or_abort(&expd[s], ph, err, abrt)
                                 : wait_or_abort(&full[s], ph, err, abrt);
        if (!ok) break;
        tc::tc_fence_after();
        const uint64_t ad = tc::desc_sw128(sA + s * A_BYTES);
        const uint64_t bd = tc::desc_sw128(sB + s * B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          tc::mma_bf16(tmem, tc::desc_advance(ad, k * 32), tc::desc_advance(bd, k * 32), idesc,
                       (kb > 0 || k > 0) ? 1u : 0u);
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(accf);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else {
    // warps 2..5: expansion of S, then the epilogue.  Row = TMEM lane.
    const int row = ((warp & 3) << 5) | lane;
    for (int kb = 0; kb < nkS; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!wait_or_abort(&full[s], ph, err, abrt)) break;
      // values arrive with the 64-byte TMA swizzle: 16-byte chunk q of a row
      // sits at chunk q ^ ((row >> 1) & 3), which spreads a quarter-warp over
      // all banks
      const unsigned char* vrow_s = sV + s * SV_BYTES + row * 64;
      const int vsw = (row >> 1) & 3;
      const uint4 ib = *reinterpret_cast<const uint4*>(sI + s * SI_BYTES + row * 16);
      const uint32_t ibw[4] = {ib.x, ib.y, ib.z, ib.w};
      unsigned char* arow = sA + s * A_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // 16 bytes of values = 4 groups = 2 chunks of 8 dense
        const uint4 v = *reinterpret_cast<const uint4*>(vrow_s + ((q ^ vsw) << 4));
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = 2 * q + h;  // dense chunk (8 columns)
          uint32_t d[4];
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const int grp = 2 * c + g;  // group within the 64-column block
            const uint32_t nib = (ibw[grp >> 2] >> (8 * (grp & 3))) & 0xFu;
            const uint32_t sel = sel_tab[nib];
            const uint32_t w = vw[2 * h + g];
            d[2 * g] = __byte_perm(w, 0u, sel & 0xFFFFu);
            d[2 * g + 1] = __byte_perm(w, 0u, sel >> 16);
          }
          *reinterpret_cast<uint4*>(arow + ((c ^ (row & 7)) << 4)) = make_uint4(d[0], d[1], d[2], d[3]);
        }
      }
      tc::fence_async_smem();
      tc::mbar_arrive(&expd[s]);
    }
    // epilogue
    if (tc::mbar_wait(accf, 0, err) && !*abrt) {
      tc::tc_fence_after();
      const int i = i0 + row;
      const uint32_t tbase = tmem + (uint32_t((warp & 3) * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        tc::tmem_ld32(tbase + c0, v);
        if (i < m) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = t0 + c0 + j;
            // streaming store: Y is written once; keep X and Z resident in L2
            if (t < T) __stcs(Y + int64_t(t) * m + i, __float2bfloat16_rn(v[j]));
          }
        }
      }
    } else {
      *abrt = 1;
    }
  }
  tc::tc_fence_before();
  tc::cta_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, BN);
  }
}

// Z = X·V : one CTA per 128 tokens, N = r16 (16..256).
__global__ void __launch_bounds__(192, 1)
    k_prefill_z(const __grid_constant__ PrefillMaps maps, __nv_bfloat16* __restrict__ Z, int n,
                int T, int r16, uint32_t* err) {
  pdl_trigger();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;
  unsigned char* sB = sA + ZSTAGES * ZA_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + ZSTAGES * ZB_MAX);
  uint64_t* empty = full + ZSTAGES;
  uint64_t* accf = empty + ZSTAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * 128;
  const int nk = (n + BK - 1) / BK;
  const uint32_t ncols = r16 <= 32 ? 32u : r16 <= 64 ? 64u : r16 <= 128 ? 128u : 256u;
  const int b_bytes = r16 * BK * 2;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ZSTAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accf, 1);
    tc::fence_mbar_init();
    tc::prefetch_tmap(&maps.xz);
    tc::prefetch_tmap(&maps.vt);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, ncols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abrt = &abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      int issued[ZSTAGES] = {0, 0, 0, 0};
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % ZSTAGES;
        const uint32_t ph = (kb / ZSTAGES) & 1;
        if (!wait_or_abort(&empty[s], ph ^ 1, err, abrt)) break;
        tc::mbar_expect_tx(&full[s], ZA_BYTES + b_bytes);
        tc::tma_load_2d(sA + s * ZA_BYTES, &maps.xz, kb * BK, t0, &full[s]);
        tc::tma_load_2d(sB + s * ZB_MAX, &maps.vt, kb * BK, 0, &full[s]);
        ++issued[s];
      }
      for (int s = 0; s < ZSTAGES; ++s)
        if (issued[s]) tc::mbar_wait(&full[s], (issued[s] - 1) & 1, err);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, r16);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % ZSTAGES;
        const uint32_t ph = (kb / ZSTAGES) & 1;
        if (!wait_or_abort(&full[s], ph, err, abrt)) break;
        tc::tc_fence_after();
        const uint64_t ad = tc::desc_sw128(sA + s * ZA_BYTES);
        const uint64_t bd = tc::desc_sw128(sB + s * ZB_MAX);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          tc::mma_bf16(tmem, tc::desc_advance(ad, k * 32), tc::desc_advance(bd, k * 32), idesc,
                       (kb > 0 || k > 0) ? 1u : 0u);
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(accf);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else {
    const int row = ((warp & 3) << 5) | lane;  // token within the tile
    if (tc::mbar_wait(accf, 0, err) && !*abrt) {
      tc::tc_fence_after();
      const int t = t0 + row;
      const uint32_t tbase = tmem + (uint32_t((warp & 3) * 32) << 16);
      for (int c0 = 0; c0 < r16; c0 += 32) {
        float v[32];
        tc::tmem_ld32(tbase + c0, v);
        if (t < T) {
          // Z as a bf16 pair: hi = bf16(z), lo = bf16(z − hi); U·(hi + lo)
          // keeps the low-rank product accurate to ~2⁻¹⁷ of |U·z|
          __nv_bfloat16* zr = Z + int64_t(t) * r16 + c0;
          __nv_bfloat16* zl = Z + int64_t(T) * r16 + int64_t(t) * r16 + c0;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            if (c0 + j < r16) {
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat16 h0 = __float2bfloat16_rn(v[j + 2 * e]);
                const __nv_bfloat16 h1 = __float2bfloat16_rn(v[j + 2 * e + 1]);
                const __nv_bfloat16 l0 = __float2bfloat16_rn(v[j + 2 * e] - __bfloat162float(h0));
                const __nv_bfloat16 l1 = __float2bfloat16_rn(v[j + 2 * e + 1] - __bfloat162float(h1));
                hw[e] = __bfloat16_as_ushort(h0) | (uint32_t(__bfloat16_as_ushort(h1)) << 16);
                lw[e] = __bfloat16_as_ushort(l0) | (uint32_t(__bfloat16_as_ushort(l1)) << 16);
              }
              *reinterpret_cast<uint4*>(zr + j) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4*>(zl + j) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
        }
      }
    } else {
      *abrt = 1;
    }
  }
  tc::tc_fence_before();
  tc::cta_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, ncols);
  }
}

// ---- sparse tensor-core prefill -------------------------------------------------
// Yᵀ tile [256 rows of W × 224 tokens]: two 128-row accumulators in TMEM share
// every X tile (half the X traffic of one 128-row tile per flop).  K-blocks of
// 64 logical columns: A = the compressed 2:4 values of all 256 rows in one TMA
// (64-byte swizzle, 32 values per row, 16 KB: a copy instruction costs a
// near-fixed time, so two 8 KB copies took about twice as long), B = X (TMA,
// 128-byte swizzle), two tcgen05.mma.sp of K = 32 per half.  Three threads
// issue the copies of a stage (warp 0 the A tile, warp 6 the B tile, warp 7 the
// metadata on its own barrier), so their copy instructions overlap.  Four warps
// put a K-block's metadata into TMEM (tcgen05.st) from a layout built at pack
// time, one 8-byte word pair per TMEM lane, and arrive on the stage's data
// barrier, so the MMA thread waits on one barrier per K-block; each MMA's
// metadata column is 4-column aligned (a requirement of the sparse MMA's
// metadata address).  The low-rank tail runs dense MMAs on
// U [256 × 32] and Z [224 × 32] K-blocks (64-byte swizzle) into the same
// accumulators.
constexpr int SP_BN = 224, SP_STAGES = 4;
constexpr int SP_A_HALF = 128 * 64;        // 128 rows × 64 bytes
constexpr int SP_A = 2 * SP_A_HALF;        // 16 KB
constexpr int SP_B = SP_BN * 128;          // 28 KB (X: 224 rows × 64 bf16)
constexpr int SP_B_Z = SP_BN * 64;         // Z: 224 rows × 32 bf16
constexpr int SP_M = 2 * 128 * 8;           // metadata of the stage: 2 halves × 128 lanes × 8 B
constexpr int SP_STAGE = SP_A + SP_B + SP_M;
constexpr int SP_SMEM = SP_STAGES * SP_STAGE + 1024 + 256;
// TMEM columns: accumulator 0 [0, SP_BN), accumulator 1 [256, 256 + SP_BN);
// metadata slots of 4 columns, one per (stage, half, MMA), in the gaps
// [SP_BN, 256) and [256 + SP_BN, 512).
constexpr uint32_t SP_ACC1_COL = 256;
constexpr int SP_GAP_SLOTS = (256 - SP_BN) / 4;  // slots in each gap
__device__ __forceinline__ uint32_t sp_meta_col(int s, int h, int i) {
  const uint32_t slot = uint32_t(s * 4 + h * 2 + i);
  return slot < uint32_t(SP_GAP_SLOTS) ? uint32_t(SP_BN) + 4u * slot
                                       : 256u + uint32_t(SP_BN) + 4u * (slot - SP_GAP_SLOTS);
}
static_assert(SP_BN % 16 == 0 && SP_BN <= 256 && SP_STAGES * 4 <= 2 * SP_GAP_SLOTS,
              "accumulators and metadata slots fit TMEM");

struct SpMaps {
  CUtensorMap x;   // X [T][n]       box {64, SP_BN} SW128
  CUtensorMap sv;  // S values [m][n/2] box {32, 256} SW64
  CUtensorMap u;   // U [m][r_pad]   box {32, 256} SW64
  CUtensorMap z;   // Z hi [T][r16]  box {32, SP_BN} SW64
  CUtensorMap zlo; // Z lo [T][r16]  box {32, SP_BN} SW64
  CUtensorMap y;   // Y [T][m]       box {256, SP_BN}, no swizzle (the epilogue's tile store)
};
// bytes of the staged output tile: [SP_BN tokens][256 rows] bf16, in the ring
constexpr int SP_Y_STAGE = SP_BN * 256 * 2;
static_assert(SP_Y_STAGE <= SP_STAGES * SP_STAGE, "output tile staging");

// Warps: 0 A copies, 1 MMA, 2-5 metadata into TMEM + epilogue, 6 B copies,
// 7 metadata copies.  A copy instruction holds its issuing thread for a
// near-fixed time whatever its size, so the three streams of copies run on
// three threads in parallel.
constexpr int SP_THREADS = 256;
__global__ void __launch_bounds__(SP_THREADS, 1)
    k_prefill_24sp(const __grid_constant__ SpMaps maps, const uint2* __restrict__ meta,
                   __nv_bfloat16* __restrict__ Y, int m, int n, int T, int r16, int ystore,
                   uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;
  unsigned char* sB = sA + SP_STAGES * SP_A;
  unsigned char* sM = sB + SP_STAGES * SP_B;
  uint64_t* full = reinterpret_cast<uint64_t*>(sM + SP_STAGES * SP_M);
  uint64_t* mload = full + SP_STAGES;  // the stage's metadata has landed
  uint64_t* empty = mload + SP_STAGES;
  uint64_t* accf = empty + SP_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntn = (T + SP_BN - 1) / SP_BN;
  const int mt = blockIdx.x / ntn, nt = blockIdx.x % ntn;
  const int i0 = mt * 256, t0 = nt * SP_BN;
  const int nkS = n / 64;
  const int nkL = (r16 + 31) / 32;
  const int nk = nkS + nkL;
  const int mtiles128 = (m + 127) / 128;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < SP_STAGES; ++s) {
      // the A and B issuers, and the 128 threads that put the stage's metadata
      // into TMEM: the MMA thread waits on this one barrier per K-block (each
      // wait on a completed phase measured 0.13-0.19 us in its loop; with a
      // second barrier for the metadata the kernel took 1.59 ms, with one
      // 1.26 ms, on the 70B layer at 4096 tokens)
      tc::mbar_init(&full[s], 2 + 128);
      tc::mbar_init(&mload[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accf, 1);
    tc::fence_mbar_init();
    tc::prefetch_tmap(&maps.x);
    tc::prefetch_tmap(&maps.sv);
    if (r16 > 0) {
      tc::prefetch_tmap(&maps.u);
      tc::prefetch_tmap(&maps.z);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abrt = &abort_flag;

  if (warp == 0 || warp >= 6) {
    // warp 0: the A tile (S values, then U); warp 6: the B tile (X, then Z hi
    // and lo); warp 7: the metadata (none for the low-rank K-blocks)
    if (lane == 0) {
      const int role = warp == 0 ? 0 : warp - 5;  // 0 A, 1 B, 2 metadata
      const uint64_t keep = tc::make_policy_evict_last();
      const uint64_t stream = tc::make_policy_evict_first();
      // the metadata issuer covers the 2:4 K-blocks only, on its own barrier,
      // so the metadata reaches TMEM while the stage's A and X are in flight
      const int nkr = role == 2 ? nkS : nk;
      uint64_t* landed = role == 2 ? mload : full;
      int kb = 0;
      for (; kb < nkr; ++kb) {
        const int s = kb % SP_STAGES;
        const uint32_t ph = (kb / SP_STAGES) & 1;
        if (!wait_or_abort(&empty[s], ph ^ 1, err, abrt)) break;
        unsigned char* a = sA + s * SP_A;
        unsigned char* b = sB + s * SP_B;
        if (role == 0) {
          tc::mbar_expect_tx(&full[s], SP_A);
          if (kb < nkS) tc::tma_load_2d_hint(a, &maps.sv, kb * 32, i0, &full[s], stream);
          else tc::tma_load_2d_hint(a, &maps.u, (kb - nkS) * 32, i0, &full[s], stream);
        } else if (role == 2) {
          // the metadata of both halves (1 KB each)
          const int mt0 = i0 / 128;
          const int nmeta = (mt0 < mtiles128) + (mt0 + 1 < mtiles128);
          tc::mbar_expect_tx(&mload[s], nmeta * 1024);
          for (int h = 0; h < 2; ++h)
            if (mt0 + h < mtiles128)
              tc::bulk_load(sM + s * SP_M + h * 1024, meta + (int64_t(mt0 + h) * nkS + kb) * 128,
                            1024, &mload[s]);
        } else if (kb < nkS) {
          tc::mbar_expect_tx(&full[s], SP_B);
          tc::tma_load_2d_hint(b, &maps.x, kb * 64, t0, &full[s], keep);
        } else {
          if (kb == nkS) pdl_wait();  // Z is written by the preceding kernel
          const int kl = kb - nkS;
          tc::mbar_expect_tx(&full[s], 2 * SP_B_Z);
          tc::tma_load_2d_hint(b, &maps.z, kl * 32, t0, &full[s], keep);
          tc::tma_load_2d_hint(b + SP_B_Z, &maps.zlo, kl * 32, t0, &full[s], keep);
        }
      }
      // drain: the last stages this thread issued have landed (the other
      // issuer's copies complete the same phases of `full`)
      for (int j = kb > SP_STAGES ? kb - SP_STAGES : 0; j < kb; ++j)
        tc::mbar_wait(&landed[j % SP_STAGES], (j / SP_STAGES) & 1, err);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_sp = tc::idesc_bf16(128, SP_BN) | (1u << 2);
      const uint32_t idesc_d = tc::idesc_bf16(128, SP_BN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % SP_STAGES;
        const uint32_t ph = (kb / SP_STAGES) & 1;
        if (!wait_or_abort(&full[s], ph, err, abrt)) break;
        tc::tc_fence_after();
        const unsigned char* a = sA + s * SP_A;
        const unsigned char* b = sB + s * SP_B;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t d = tmem + (h ? SP_ACC1_COL : 0u);
          const uint64_t ad = tc::desc_sw64(a + h * SP_A_HALF);
          if (kb < nkS) {
            const uint64_t bd = tc::desc_sw128(b);
#pragma unroll
            for (int i = 0; i < 2; ++i)
              tc::mma_bf16_sp(d, tc::desc_advance(ad, 32 * i), tc::desc_advance(bd, 64 * i),
                              tmem + sp_meta_col(s, h, i), idesc_sp,
                              (kb > 0 || i > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int part = 0; part < 2; ++part) {  // Z hi, then Z lo
              const uint64_t bd = tc::desc_sw64(b + part * SP_B_Z);
#pragma unroll
              for (int i = 0; i < 2; ++i)
                tc::mma_bf16(d, tc::desc_advance(ad, 32 * i), tc::desc_advance(bd, 32 * i), idesc_d,
                             1u);
            }
          }
        }
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(accf);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp < 6) {
    // warps 2..5: metadata into TMEM, then the epilogue.  TMEM lane = L.
    const int L = ((warp & 3) << 5) | lane;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % SP_STAGES;
      const uint32_t ph = (kb / SP_STAGES) & 1;
      if (kb >= nkS) {
        // no metadata: arrive once the stage's previous MMAs are done, so the
        // arrival counts towards this K-block's phase
        if (!wait_or_abort(&empty[s], ph ^ 1, err, abrt)) break;
        tc::mbar_arrive(&full[s]);
        continue;
      }
      // the stage's metadata has landed, so its previous MMAs (the last
      // readers of these TMEM slots) are done
      if (!wait_or_abort(&mload[s], ph, err, abrt)) break;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int mt128 = i0 / 128 + h;
        uint2 w = make_uint2(0x44444444u, 0x44444444u);  // rows past m: a valid pattern, zero values
        if (mt128 < mtiles128) w = *reinterpret_cast<const uint2*>(sM + s * SP_M + h * 1024 + L * 8);
        tc::tmem_st1(tmem + lane_base + sp_meta_col(s, h, 0), w.x);
        tc::tmem_st1(tmem + lane_base + sp_meta_col(s, h, 1), w.y);
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(&full[s]);
    }
    if (tc::mbar_wait(accf, 0, err) && !*abrt) {
      tc::tc_fence_after();
      if (ystore) {
        // The tile, rounded to bf16, into shared memory as [token][row] (the ring
        // is idle: every copy was consumed before the last MMAs), then one tiled
        // store; rows past m and tokens past T are not written.  Scattered 2-byte
        // stores straight from registers took ~13 µs per tile.
        __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
#pragma unroll 1
          for (int c0 = 0; c0 < SP_BN; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tmem + lane_base + (h ? SP_ACC1_COL : 0u) + c0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) stg[(c0 + j) * 256 + 128 * h + L] = __float2bfloat16_rn(v[j]);
          }
        }
        tc::fence_async_smem();
        asm volatile("barrier.sync 1, 128;" ::: "memory");  // the four epilogue warps
        if (L == 0) {
          tc::tma_store_2d(&maps.y, stg, i0, t0);
          tc::bulk_commit();
          tc::bulk_wait_read_all();  // the CTA's shared memory is read before it ends
        }
      } else {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int i = i0 + 128 * h + L;
#pragma unroll 1
          for (int c0 = 0; c0 < SP_BN; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tmem + lane_base + (h ? SP_ACC1_COL : 0u) + c0, v);
            if (i < m) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int t = t0 + c0 + j;
                if (c0 + j < SP_BN && t < T) __stcs(Y + int64_t(t) * m + i, __float2bfloat16_rn(v[j]));
              }
            }
          }
        }
      }
    } else {
      *abrt = 1;
    }
  }
  tc::tc_fence_before();
  tc::cta_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---- sparse tensor-core prefill on CTA pairs -------------------------------------
// A cluster of two CTAs shares each MMA (cta_group::2, M = 256): CTA r of the
// pair stages its own 128 rows of A and half of the X tile (B is split along
// N), and its TMEM holds the accumulator rows of its A half.  Two such MMAs
// (pair rows [0, 256) and [256, 512) of the tile) share every X tile, so a
// pair tile is 512 rows of W × 192 tokens and each SM loads, per K-block,
// 256 rows of A and 96 tokens of X: ~1.5× the MMA work per byte of the
// single-CTA 256 × 192 tile, with deeper loads in flight.
//   Per K-block both CTAs' loads count on the even CTA's `full` barrier; the
// even CTA's MMA thread waits on it and on `mready` (the 2:4 metadata of both
// CTAs is in TMEM), issues the MMAs and commits to `empty` in both CTAs.  The
// metadata warps load their 2 KB of metadata per K-block straight from global
// memory, ahead of the MMAs, into one of NSLOT slot sets; a slot set is
// reused once the MMA NSLOT K-blocks back has completed (`empty`).
constexpr int P2_BN = 192, P2_BNH = P2_BN / 2;  // tokens of a pair tile / staged per CTA
constexpr int P2_STAGES = 8, P2_NSLOT = 8;
constexpr int P2_A_HALF = 128 * 64;             // 128 rows × 64 bytes
constexpr int P2_A = 2 * P2_A_HALF;             // 16 KB: this CTA's rows of both MMAs
constexpr int P2_B = P2_BNH * 128;              // 12 KB: X, 96 tokens × 64 bf16
constexpr int P2_B_Z = P2_BNH * 64;             // Z hi / lo: 96 tokens × 32 bf16
constexpr int P2_STAGE = P2_A + P2_B;
constexpr int P2_SMEM = P2_STAGES * P2_STAGE + 1024 + 256;
// TMEM: accumulators [0, 192) and [256, 448); metadata slots of 4 columns,
// k = 4·set + 2·h + i: 16 in [192, 256), 16 in [448, 512).
constexpr uint32_t P2_ACC1_COL = 256;
__device__ __forceinline__ uint32_t p2_meta_col(int set, int h, int i) {
  const uint32_t k = uint32_t(set * 4 + h * 2 + i);
  return k < 16 ? 192u + 4u * k : 448u + 4u * (k - 16u);
}
static_assert(P2_NSLOT * 4 == 32, "metadata slots");
static_assert(P2_STAGE % 1024 == 0 && P2_A % 1024 == 0, "tile alignment");

// Barrier 1 over the four metadata warps (128 threads), returning the OR of
// `v` over them, so that they take every branch together.
__device__ __forceinline__ int meta_bar_or(int v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return int(r);
}

struct PairMaps {
  CUtensorMap x;    // X [T][n]         box {64, 96} SW128
  CUtensorMap sv;   // S values [m][n/2] box {32, 128} SW64
  CUtensorMap u;    // U [m][r_pad]     box {32, 128} SW64
  CUtensorMap z;    // Z hi [T][r16]    box {32, 96} SW64
  CUtensorMap zlo;  // Z lo [T][r16]    box {32, 96} SW64
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    k_prefill_24sp2(const __grid_constant__ PairMaps maps, const uint2* __restrict__ meta,
                    __nv_bfloat16* __restrict__ Y, int m, int n, int T, int r16, uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P2_STAGES * P2_STAGE);
  uint64_t* empty = full + P2_STAGES;
  uint64_t* mready = empty + P2_STAGES;
  uint64_t* accf = mready + P2_NSLOT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int ntn = (T + P2_BN - 1) / P2_BN;
  const int mt = pair / ntn, nt = pair % ntn;
  const int i0 = mt * 512, t0 = nt * P2_BN;
  const int nkS = n / 64;
  const int nkL = (r16 + 31) / 32;
  const int nk = nkS + nkL;
  const int mtiles128 = (m + 127) / 128;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < P2_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < P2_NSLOT; ++j) tc::mbar_init(&mready[j], 2);  // one arrival per CTA
    tc::mbar_init(accf, 1);
    tc::fence_mbar_init();
    tc::prefetch_tmap(&maps.x);
    tc::prefetch_tmap(&maps.sv);
    if (r16 > 0) {
      tc::prefetch_tmap(&maps.u);
      tc::prefetch_tmap(&maps.z);
      tc::prefetch_tmap(&maps.zlo);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc2(tmem_slot, 512);
    tc::tmem_relinquish2();
  }
  tc::tc_fence_before();
  tc::cluster_sync();  // both CTAs' barriers and TMEM are ready
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abrt = &abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t keep = tc::make_policy_evict_last();
      const uint64_t stream = tc::make_policy_evict_first();
      const int rowA0 = i0 + 128 * int(rank), rowA1 = rowA0 + 256;
      const int tB = t0 + P2_BNH * int(rank);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % P2_STAGES;
        const uint32_t ph = (kb / P2_STAGES) & 1;
        if (!wait_or_abort(&empty[s], ph ^ 1, err, abrt)) break;
        unsigned char* a = smem + s * P2_STAGE;
        unsigned char* b = a + P2_A;
        if (kb < nkS) {
          if (leader) tc::mbar_expect_tx(&full[s], 2 * (P2_A + P2_B));
          tc::tma_load_2d_pair(a, &maps.sv, kb * 32, rowA0, &full[s], stream);
          tc::tma_load_2d_pair(a + P2_A_HALF, &maps.sv, kb * 32, rowA1, &full[s], stream);
          tc::tma_load_2d_pair(b, &maps.x, kb * 64, tB, &full[s], keep);
        } else {
          if (kb == nkS) pdl_wait();  // Z is written by the preceding kernel
          const int kl = kb - nkS;
          if (leader) tc::mbar_expect_tx(&full[s], 2 * (P2_A + 2 * P2_B_Z));
          tc::tma_load_2d_pair(a, &maps.u, kl * 32, rowA0, &full[s], stream);
          tc::tma_load_2d_pair(a + P2_A_HALF, &maps.u, kl * 32, rowA1, &full[s], stream);
          tc::tma_load_2d_pair(b, &maps.z, kl * 32, tB, &full[s], keep);
          tc::tma_load_2d_pair(b + P2_B_Z, &maps.zlo, kl * 32, tB, &full[s], keep);
        }
      }
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc_sp = tc::idesc_bf16(256, P2_BN) | (1u << 2);
      const uint32_t idesc_d = tc::idesc_bf16(256, P2_BN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % P2_STAGES;
        const uint32_t ph = (kb / P2_STAGES) & 1;
        if (!wait_or_abort(&full[s], ph, err, abrt)) break;
        const int set = kb % P2_NSLOT;
        if (kb < nkS && !wait_or_abort(&mready[set], (kb / P2_NSLOT) & 1, err, abrt)) break;
        tc::tc_fence_after();
        const unsigned char* a = smem + s * P2_STAGE;
        const unsigned char* b = a + P2_A;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t d = tmem + (h ? P2_ACC1_COL : 0u);
          const uint64_t ad = tc::desc_sw64(a + h * P2_A_HALF);
          if (kb < nkS) {
            const uint64_t bd = tc::desc_sw128(b);
#pragma unroll
            for (int i = 0; i < 2; ++i)
              tc::mma_bf16_sp_pair(d, tc::desc_advance(ad, 32 * i), tc::desc_advance(bd, 64 * i),
                                   tmem + p2_meta_col(set, h, i), idesc_sp,
                                   (kb > 0 || i > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int part = 0; part < 2; ++part) {  // Z hi, then Z lo
              const uint64_t bd = tc::desc_sw64(b + part * P2_B_Z);
#pragma unroll
              for (int i = 0; i < 2; ++i)
                tc::mma_bf16_pair(d, tc::desc_advance(ad, 32 * i), tc::desc_advance(bd, 32 * i),
                                  idesc_d, 1u);
            }
          }
        }
        tc::mma_commit_pair(&empty[s]);
      }
      tc::mma_commit_pair(accf);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else {
    // warps 2..5: metadata into TMEM ahead of the MMAs, then the epilogue
    const int L = ((warp & 3) << 5) | lane;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t mready0 = tc::mapa(tc::smem_u32(&mready[0]), 0);
    const int mtA = i0 / 128 + int(rank);  // 128-row tiles of this CTA: mtA, mtA + 2
    auto load_meta = [&](int kb, int h) {
      const int mt128 = mtA + 2 * h;
      uint2 w = make_uint2(0x44444444u, 0x44444444u);  // rows past m: valid pattern, zero values
      if (kb < nkS && mt128 < mtiles128) w = __ldg(meta + (int64_t(mt128) * nkS + kb) * 128 + L);
      return w;
    };
    constexpr int D = 4;  // K-blocks of metadata loaded ahead
    uint2 ring[D][2];
#pragma unroll
    for (int d = 0; d < D; ++d) {
      ring[d][0] = load_meta(d, 0);
      ring[d][1] = load_meta(d, 1);
    }
    bool ok = true;
    for (int kb0 = 0; kb0 < nkS && ok; kb0 += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int kb = kb0 + d;
        if (kb >= nkS || !ok) break;
        const int set = kb % P2_NSLOT;
        // the MMA that last used this slot set has completed (one thread
        // waits; the four warps decide together whether to go on)
        int fail = 0;
        if (kb >= P2_NSLOT && L == 0) {
          const int kp = kb - P2_NSLOT;
          fail = !wait_or_abort(&empty[kp % P2_STAGES], (kp / P2_STAGES) & 1, err, abrt);
        }
        if (meta_bar_or(fail)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tc::tmem_st1(tmem + lane_base + p2_meta_col(set, h, 0), ring[d][h].x);
          tc::tmem_st1(tmem + lane_base + p2_meta_col(set, h, 1), ring[d][h].y);
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
        // the four warps' stores are done: one arrival per CTA (cluster-scope
        // release), not one per thread
        asm volatile("barrier.sync 1, 128;" ::: "memory");
        if (L == 0) tc::mbar_arrive_cluster(mready0 + uint32_t(set) * 8u);
        ring[d][0] = load_meta(kb + D, 0);
        ring[d][1] = load_meta(kb + D, 1);
      }
    }
    if (tc::mbar_wait(accf, 0, err) && !*abrt) {
      tc::tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int i = i0 + 256 * h + 128 * int(rank) + L;
#pragma unroll 1
        for (int c0 = 0; c0 < P2_BN; c0 += 32) {
          float v[32];
          tc::tmem_ld32(tmem + lane_base + (h ? P2_ACC1_COL : 0u) + c0, v);
          if (i < m) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = t0 + c0 + j;
              if (t < T) __stcs(Y + int64_t(t) * m + i, __float2bfloat16_rn(v[j]));
            }
          }
        }
      }
    } else {
      *abrt = 1;
    }
  }
  tc::tc_fence_before();
  tc::cluster_sync_any();  // the pair is done with its TMEM and barriers
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc2(tmem, 512);
  }
}

// ---- host: tensor maps through the driver entry point (no libcuda link) -----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D row-major map: `rows` × `cols` elements, box {box_cols, box_rows}.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, int64_t rows,
              int64_t cols, int64_t row_stride_elems, int box_cols, int box_rows,
              CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(row_stride_elems * esize)};
  cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base,
                  int64_t rows, int64_t cols, int64_t row_stride_elems, int box_cols,
                  int box_rows, CUtensorMapSwizzle sw) {
  return make_map(map, dt, esize, base, rows, cols, row_stride_elems, box_cols, box_rows, sw);
}
bool make_tmap_kblocks(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                       int box_rows, int box_kblocks) {
  const EncodeTiledFn fn = encode_fn();
  if (!fn || cols % 64 != 0) return false;
  cuuint64_t dims[3] = {64, cuuint64_t(rows), cuuint64_t(cols / 64)};
  cuuint64_t strides[2] = {cuuint64_t(cols * 2), 128};
  cuuint32_t box[3] = {64, cuuint32_t(box_rows), cuuint32_t(box_kblocks)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool tmap_available() { return encode_fn() != nullptr; }

// Z workspace and Vt come from the handle (Vt built when the factors are packed).
// Pair tiles hold 192 tokens: below a few tiles of tokens the single-CTA
// kernel wastes less of its tile.
constexpr int64_t kPairMinTokens = 512;
// HSL_PREFILL_PAIRS=1 selects the CTA-pair kernel.  It is exact (the parity
// tests cover it) but measured slower than the single-CTA kernel on the 70B
// layer (3.2 ms, measured against 1.66 ms for the single-CTA kernel of that time;
// that kernel now takes 1.15 ms), so it is not the default.
bool prefill_pairs_enabled() {
  const char* e = std::getenv("HSL_PREFILL_PAIRS");
  return e != nullptr && e[0] == '1';
}

// Z = X·V as a bf16 (hi, lo) pair into h.zpre ([2][T][r16]); the kernel
// triggers programmatic dependent launch at its start.
hsl_status prefill_z_run(Handle& h, const void* X, int64_t T, cudaStream_t s) {
  const int r16 = int(round_up(h.r, 16));
  if (r16 == 0) return HSL_OK;
  if (r16 > 256) return HSL_ERR_UNSUPPORTED;
  if (hsl_status e = ensure(h.zpre, size_t(T) * r16 * 2 * 2, "prefill Z (hi, lo)")) return e;
  PrefillMaps zm;
  memset(&zm, 0, sizeof(zm));
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&zm.xz, BF, 2, X, T, h.n, h.n, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&zm.vt, BF, 2, h.Vt.p, r16, h.n, h.n, 64, r16, CU_TENSOR_MAP_SWIZZLE_128B)) {
    set_message("tensor map encoding failed");
    return HSL_ERR_CUDA;
  }
  if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_prefill_z), Z_SMEM))
    return cuda_fail(e, "prefill z smem attribute");
  k_prefill_z<<<unsigned((T + 127) / 128), 192, Z_SMEM, s>>>(
      zm, static_cast<__nv_bfloat16*>(h.zpre.p), int(h.n), int(T), r16,
      static_cast<uint32_t*>(h.err.p));
  note_launch();
  return cuda_fail(cudaGetLastError(), "prefill z launch");
}

bool prefill_supported(const Handle& h, const void* X) {
  return h.fmt == HSL_FMT_NM24 && h.dtype == HSL_BF16 && h.n % 64 == 0 &&
         (reinterpret_cast<uintptr_t>(X) % 16) == 0 && encode_fn() != nullptr;
}

hsl_status apply_prefill_run(Handle& h, const void* X, void* Y, int64_t T, cudaStream_t s) {
  const int r16 = int(round_up(h.r, 16));
  if (r16 > 256) return HSL_ERR_UNSUPPORTED;
  const int64_t m = h.m, n = h.n;
  if (r16 > 0) {
    if (hsl_status e = ensure(h.zpre, size_t(T) * r16 * 2 * 2, "prefill Z (hi, lo)")) return e;
  }
  uint32_t* err0 = static_cast<uint32_t*>(h.err.p);
  if (h.pmeta_tc.p && std::getenv("HSL_PREFILL_EXPAND") == nullptr) {
    // sparse tensor-core path
    SpMaps sm;
    memset(&sm, 0, sizeof(sm));
    const auto BFs = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    bool ok = make_map(&sm.x, BFs, 2, X, T, n, n, 64, SP_BN, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&sm.sv, BFs, 2, h.nm_val.p, m, n / 2, n / 2, 32, 256,
                       CU_TENSOR_MAP_SWIZZLE_64B);
    // the epilogue's tiled store needs 16-byte row pitch and base
    const int ystore = (m % 8 == 0 && reinterpret_cast<uintptr_t>(Y) % 16 == 0) ? 1 : 0;
    if (ok && ystore)
      ok = make_map(&sm.y, BFs, 2, Y, T, m, m, 256, SP_BN, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && r16 > 0)
      ok = make_map(&sm.u, BFs, 2, h.U.p, m, h.r_pad, h.r_pad, 32, 256, CU_TENSOR_MAP_SWIZZLE_64B) &&
           make_map(&sm.z, BFs, 2, h.zpre.p, T, r16, r16, 32, SP_BN, CU_TENSOR_MAP_SWIZZLE_64B) &&
           make_map(&sm.zlo, BFs, 2, static_cast<__nv_bfloat16*>(h.zpre.p) + T * r16, T, r16, r16,
                    32, SP_BN, CU_TENSOR_MAP_SWIZZLE_64B);
    PrefillMaps zm;
    memset(&zm, 0, sizeof(zm));
    if (ok && r16 > 0)
      ok = make_map(&zm.xz, BFs, 2, X, T, n, n, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map(&zm.vt, BFs, 2, h.Vt.p, r16, n, n, 64, r16, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) {
      set_message("tensor map encoding failed");
      return HSL_ERR_CUDA;
    }
    if (r16 > 0) {
      if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_prefill_z), Z_SMEM))
        return cuda_fail(e, "prefill z smem attribute");
      k_prefill_z<<<unsigned((T + 127) / 128), 192, Z_SMEM, s>>>(
          zm, static_cast<__nv_bfloat16*>(h.zpre.p), int(n), int(T), r16, err0);
      note_launch();
      if (hsl_status e = cuda_fail(cudaGetLastError(), "prefill z launch")) return e;
    }
    if (prefill_pairs_enabled() && T >= kPairMinTokens) {
      // CTA pairs: 512 rows × 192 tokens per pair
      PairMaps pm;
      memset(&pm, 0, sizeof(pm));
      bool okp = make_map(&pm.x, BFs, 2, X, T, n, n, 64, P2_BNH, CU_TENSOR_MAP_SWIZZLE_128B) &&
                 make_map(&pm.sv, BFs, 2, h.nm_val.p, m, n / 2, n / 2, 32, 128,
                          CU_TENSOR_MAP_SWIZZLE_64B);
      if (okp && r16 > 0)
        okp = make_map(&pm.u, BFs, 2, h.U.p, m, h.r_pad, h.r_pad, 32, 128,
                       CU_TENSOR_MAP_SWIZZLE_64B) &&
              make_map(&pm.z, BFs, 2, h.zpre.p, T, r16, r16, 32, P2_BNH, CU_TENSOR_MAP_SWIZZLE_64B) &&
              make_map(&pm.zlo, BFs, 2, static_cast<__nv_bfloat16*>(h.zpre.p) + T * r16, T, r16,
                       r16, 32, P2_BNH, CU_TENSOR_MAP_SWIZZLE_64B);
      if (!okp) {
        set_message("tensor map encoding failed");
        return HSL_ERR_CUDA;
      }
      if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_prefill_24sp2), P2_SMEM))
        return cuda_fail(e, "prefill smem attribute");
      const int64_t pairs = ((m + 511) / 512) * ((T + P2_BN - 1) / P2_BN);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(unsigned(2 * pairs));
      cfg.blockDim = dim3(192);
      cfg.dynamicSmemBytes = P2_SMEM;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = r16 > 0 ? 1 : 0;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      note_launch();
      return cuda_fail(cudaLaunchKernelEx(&cfg, k_prefill_24sp2, pm,
                                          static_cast<const uint2*>(h.pmeta_tc.p),
                                          static_cast<__nv_bfloat16*>(Y), int(m), int(n), int(T),
                                          r16, err0),
                       "pair prefill launch");
    }
    if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_prefill_24sp), SP_SMEM))
      return cuda_fail(e, "prefill smem attribute");
    const int64_t tiles = ((m + 255) / 256) * ((T + SP_BN - 1) / SP_BN);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(tiles));
    cfg.blockDim = dim3(SP_THREADS);
    cfg.dynamicSmemBytes = SP_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = r16 > 0 ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    note_launch();
    return cuda_fail(cudaLaunchKernelEx(&cfg, k_prefill_24sp, sm,
                                        static_cast<const uint2*>(h.pmeta_tc.p),
                                        static_cast<__nv_bfloat16*>(Y), int(m), int(n), int(T),
                                        r16, ystore, err0),
                     "sparse prefill launch");
  }
  PrefillMaps maps;
  memset(&maps, 0, sizeof(maps));
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B, NO = CU_TENSOR_MAP_SWIZZLE_NONE;
  bool ok = make_map(&maps.x, BF, 2, X, T, n, n, 64, 256, SW) &&
            make_map(&maps.xz, BF, 2, X, T, n, n, 64, 128, SW) &&
            make_map(&maps.sv, BF, 2, h.nm_val.p, m, n / 2, n / 2, 32, 128,
                     CU_TENSOR_MAP_SWIZZLE_64B) &&
            make_map(&maps.si, U8, 1, h.nm_idx.p, m, n / 4, n / 4, 16, 128, NO);
  if (ok && r16 > 0)
    ok = make_map(&maps.u, BF, 2, h.U.p, m, h.r_pad, h.r_pad, 64, 128, SW) &&
         make_map(&maps.z, BF, 2, h.zpre.p, T, r16, r16, 64, 256, SW) &&
         make_map(&maps.vt, BF, 2, h.Vt.p, r16, n, n, 64, r16, SW);
  if (!ok) {
    set_message("tensor map encoding failed");
    return HSL_ERR_CUDA;
  }
  uint32_t* err = static_cast<uint32_t*>(h.err.p);
  if (r16 > 0) {
    if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_prefill_z), Z_SMEM))
      return cuda_fail(e, "prefill z smem attribute");
    k_prefill_z<<<unsigned((T + 127) / 128), 192, Z_SMEM, s>>>(
        maps, static_cast<__nv_bfloat16*>(h.zpre.p), int(n), int(T), r16, err);
    note_launch();
    if (hsl_status e = cuda_fail(cudaGetLastError(), "prefill z launch")) return e;
  }
  if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_prefill_24), PREFILL_SMEM))
    return cuda_fail(e, "prefill smem attribute");
  const int64_t tiles = ((m + BM - 1) / BM) * ((T + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(tiles));
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = PREFILL_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = r16 > 0 ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cuda_fail(cudaLaunchKernelEx(&cfg, k_prefill_24, maps,
                                      static_cast<__nv_bfloat16*>(Y), int(m), int(n), int(T),
                                      r16, err),
                   "prefill launch");
}

}  // namespace hsl
