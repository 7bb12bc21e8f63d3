// Large-batch apply of an unstructured (CSR) S on the tensor cores: each
// 64-column block of S is decompressed into shared memory as a dense tile.
//
// "Hierarchical Sparse + Low-Rank Compression of LLMs", §Implementation and
// operational patterns (operating pattern 3, dynamic decompression): keep the
// layer factored in memory and decompress on the fly where latency matters;
// the same section notes that large batches gain less from sparsity, being
// compute-bound.  At thousands of tokens the CUDA-core CSR kernel would stream
// S once per 16 tokens; here every CTA owns a Yᵀ tile of 256 rows × 256 tokens
// (two 128-row TMEM accumulators sharing every X block, which halves the X
// bytes per FLOP of a 128-row tile) and runs the dense 5th-generation MMA over
// S's rows block by block:
//
//   warp 0 lane 0   TMA of the X block [256 tokens × 64] (128-byte swizzle);
//                   for the low-rank tail, TMA of U [128 × 64] and of Z hi or
//                   Z lo [256 × 64] (Z = X·V from k_prefill_z, a bf16 pair).
//   warps 2-9       one row of the tile per thread: zero the row of the A tile
//                   (128-byte swizzle) and drop in the row's entries whose
//                   column falls in the block, from a register cursor over the
//                   packed row (16-bit columns, ascending, the next 8 entries
//                   prefetched), then hand the tile to the MMA warp.
//   warp 1 lane 0   tcgen05.mma (M = 128, N = 256, K = 16 × 4 per block, per
//                   half) into two fp32 TMEM accumulators: S·Xᵀ, then
//                   U·Z_hiᵀ + U·Z_loᵀ.
//   warps 2-9       epilogue: tcgen05.ld, round to bf16, Y[t][i].
// The work executed is the dense product (2·T·m·n) plus the low-rank term;
// the decompression costs shared-memory stores only.  Every wait is bounded.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hsl {
namespace {

constexpr int PC_BM = 256, PC_BN = 256, PC_BK = 64, PC_STAGES = 3;
constexpr int PC_THREADS = 320;        // 10 warps: copies, MMA, 8 × decompression + epilogue
constexpr int PC_AH = 128 * 128;       // 16 KB: 128 rows × 64 bf16 (one accumulator's rows)
constexpr int PC_A = 2 * PC_AH;        // both halves of the 256-row tile
constexpr int PC_B = PC_BN * 128;      // 32 KB: 256 tokens × 64 bf16
constexpr int PC_STAGE = PC_A + PC_B;
constexpr int PC_SMEM = PC_STAGES * PC_STAGE + 1024 + 256;
constexpr uint32_t PC_ACC1 = 256;      // TMEM column of the second accumulator

struct PcMaps {
  CUtensorMap x;    // X [T][n]         box {64, 256} SW128
  CUtensorMap u;    // U [m][r_pad]     box {64, 128} SW128
  CUtensorMap zhi;  // Z hi [T][r16]    box {64, 256} SW128
  CUtensorMap zlo;  // Z lo [T][r16]    box {64, 256} SW128
  CUtensorMap y;    // Y [T][m]         box {256, 256}, no swizzle (the epilogue's tile store)
};
static_assert(PC_BN * PC_BM * 2 <= PC_STAGES * PC_STAGE, "output tile staging");

__device__ __forceinline__ bool pc_wait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                        volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (tc::mbar_wait(bar, parity, err)) return true;
  *abort_flag = 1;
  return false;
}

__global__ void __launch_bounds__(PC_THREADS, 1)
    k_prefill_csr(const __grid_constant__ PcMaps maps, const int32_t* __restrict__ prow,
                  const uint16_t* __restrict__ pcol, const uint16_t* __restrict__ pval,
                  __nv_bfloat16* __restrict__ Y, int m, int n, int T, int r16, int ystore,
                  uint32_t* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + PC_STAGES * PC_STAGE);
  uint64_t* empty = full + PC_STAGES;
  uint64_t* accf = empty + PC_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntn = (T + PC_BN - 1) / PC_BN;
  const int mt = blockIdx.x / ntn, nt = blockIdx.x % ntn;
  const int i0 = mt * PC_BM, t0 = nt * PC_BN;
  const int nkS = (n + PC_BK - 1) / PC_BK;
  const int nkL = r16 > 0 ? 2 * ((r16 + PC_BK - 1) / PC_BK) : 0;
  const int nk = nkS + nkL;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < PC_STAGES; ++s) {
      // the copy issuer and the 256 threads that decompress the stage's A tile
      // (none for the low-rank K-blocks, but they arrive all the same): the MMA
      // thread waits on this one barrier per K-block
      tc::mbar_init(&full[s], 1 + 256);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accf, 1);
    tc::fence_mbar_init();
    tc::prefetch_tmap(&maps.x);
    if (r16 > 0) {
      tc::prefetch_tmap(&maps.u);
      tc::prefetch_tmap(&maps.zhi);
      tc::prefetch_tmap(&maps.zlo);
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

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t keep = tc::make_policy_evict_last();
      const uint64_t stream = tc::make_policy_evict_first();
      int issued[PC_STAGES] = {0, 0, 0};
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % PC_STAGES;
        const uint32_t ph = (kb / PC_STAGES) & 1;
        if (!pc_wait(&empty[s], ph ^ 1, err, abrt)) break;
        unsigned char* a = smem + s * PC_STAGE;
        unsigned char* b = a + PC_A;
        if (kb < nkS) {
          tc::mbar_expect_tx(&full[s], PC_B);
          tc::tma_load_2d_hint(b, &maps.x, kb * PC_BK, t0, &full[s], keep);
        } else {
          if (kb == nkS) pdl_wait();  // Z is written by the preceding kernel
          const int lr = kb - nkS, rb = lr >> 1;
          tc::mbar_expect_tx(&full[s], PC_A + PC_B);
          tc::tma_load_2d_hint(a, &maps.u, rb * PC_BK, i0, &full[s], stream);
          tc::tma_load_2d_hint(a + PC_AH, &maps.u, rb * PC_BK, i0 + 128, &full[s], stream);
          tc::tma_load_2d_hint(b, (lr & 1) ? &maps.zlo : &maps.zhi, rb * PC_BK, t0, &full[s], keep);
        }
        ++issued[s];
      }
      for (int s = 0; s < PC_STAGES; ++s)
        if (issued[s]) tc::mbar_wait(&full[s], (issued[s] - 1) & 1, err);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, PC_BN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % PC_STAGES;
        const uint32_t ph = (kb / PC_STAGES) & 1;
        if (!pc_wait(&full[s], ph, err, abrt)) break;
        tc::tc_fence_after();
        unsigned char* a = smem + s * PC_STAGE;
        const uint64_t bd = tc::desc_sw128(a + PC_A);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint64_t ad = tc::desc_sw128(a + h * PC_AH);
#pragma unroll
          for (int k = 0; k < PC_BK / 16; ++k)
            tc::mma_bf16(tmem + (h ? PC_ACC1 : 0u), tc::desc_advance(ad, k * 32),
                         tc::desc_advance(bd, k * 32), idesc, (kb > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(accf);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else {
    // decompression: thread R owns row i0 + R of the tile; rows 0..127 belong to
    // the first accumulator, 128..255 to the second (TMEM lane R mod 128; warp
    // w may reach TMEM lanes 32·(w mod 4) onwards)
    const int half = warp >= 6 ? 1 : 0;
    const int L = ((warp & 3) << 5) | lane;
    const int R = half * 128 + L;
    const int i = i0 + R;
    int32_t e = 0, e_end = 0;
    if (i < m) {
      e = prow[i];
      e_end = prow[i + 1];
    }
    // the current 8 entries (cols, vals) and the next 8, prefetched
    uint4 cc = make_uint4(0, 0, 0, 0), cv = cc, nc = cc, nv = cc;
    if (e < e_end) {
      cc = ld_stream16(pcol + e);
      cv = ld_stream16(pval + e);
    }
    if (e + 8 < e_end) {
      nc = ld_stream16(pcol + e + 8);
      nv = ld_stream16(pval + e + 8);
    }
    int pos = 0;  // next unread entry of the current 8
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % PC_STAGES;
      const uint32_t ph = (kb / PC_STAGES) & 1;
      // the MMAs of this stage's previous use have read its A tile (and so this
      // arrival counts towards this K-block's phase)
      if (!pc_wait(&empty[s], ph ^ 1, err, abrt)) break;
      if (kb >= nkS) {  // a low-rank K-block: its A tile (U) comes by copy
        tc::mbar_arrive(&full[s]);
        continue;
      }
      unsigned char* arow = smem + s * PC_STAGE + half * PC_AH + (L >> 3) * 1024 + (L & 7) * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(arow + c * 16) = make_uint4(0, 0, 0, 0);
      const int k0 = kb * PC_BK, kend = k0 + PC_BK;
      while (e < e_end) {
        const uint32_t cw[4] = {cc.x, cc.y, cc.z, cc.w};
        const uint32_t vw[4] = {cv.x, cv.y, cv.z, cv.w};
        bool block_done = false;
        for (; pos < 8; ++pos) {
          const int col = int((cw[pos >> 1] >> ((pos & 1) * 16)) & 0xFFFFu);
          if (col >= kend) {
            block_done = true;
            break;
          }
          const int j = col - k0;  // ascending columns: col ≥ k0 here
          if (j >= 0) {
            const uint16_t v = uint16_t((vw[pos >> 1] >> ((pos & 1) * 16)) & 0xFFFFu);
            *reinterpret_cast<uint16_t*>(arow + ((((j >> 3) ^ (L & 7)) << 4) | ((j & 7) << 1))) = v;
          }
        }
        if (block_done) break;
        // the 8 entries are used up: move to the prefetched ones, fetch the next
        e += 8;
        pos = 0;
        cc = nc;
        cv = nv;
        if (e + 8 < e_end) {
          nc = ld_stream16(pcol + e + 8);
          nv = ld_stream16(pval + e + 8);
        }
      }
      tc::fence_async_smem();
      tc::mbar_arrive(&full[s]);
    }
    // epilogue
    if (tc::mbar_wait(accf, 0, err) && !*abrt) {
      tc::tc_fence_after();
      const uint32_t tbase = tmem + (uint32_t((warp & 3) * 32) << 16) + (half ? PC_ACC1 : 0u);
      if (ystore) {
        // the rounded tile into the idle ring as [token][row], then one tiled
        // store (rows past m and tokens past T are not written)
        __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem);
#pragma unroll 1
        for (int c0 = 0; c0 < PC_BN; c0 += 32) {
          float v[32];
          tc::tmem_ld32(tbase + c0, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[(c0 + j) * PC_BM + R] = __float2bfloat16_rn(v[j]);
        }
        tc::fence_async_smem();
        asm volatile("barrier.sync 1, 256;" ::: "memory");  // the eight epilogue warps
        if (R == 0) {
          tc::tma_store_2d(&maps.y, stg, i0, t0);
          tc::bulk_commit();
          tc::bulk_wait_read_all();  // the CTA's shared memory is read before it ends
        }
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < PC_BN; c0 += 32) {
          float v[32];
          tc::tmem_ld32(tbase + c0, v);
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
  tc::cta_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool prefill_csr_supported(const Handle& h, const void* X) {
  return h.fmt == HSL_FMT_CSR && h.dtype == HSL_BF16 && h.csr_ascending && h.n % 8 == 0 &&
         h.r <= 256 && (reinterpret_cast<uintptr_t>(X) % 16) == 0 && tmap_available();
}

hsl_status apply_prefill_csr_run(Handle& h, const void* X, void* Y, int64_t T, cudaStream_t s) {
  const int r16 = int(round_up(h.r, 16));
  const int64_t m = h.m, n = h.n;
  if (hsl_status e = prefill_z_run(h, X, T, s)) return e;
  PcMaps maps;
  memset(&maps, 0, sizeof(maps));
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = make_tmap_2d(&maps.x, BF, 2, X, T, n, n, 64, PC_BN, SW);
  // the epilogue's tiled store needs 16-byte row pitch and base
  const int ystore = (m % 8 == 0 && reinterpret_cast<uintptr_t>(Y) % 16 == 0) ? 1 : 0;
  if (ok && ystore)
    ok = make_tmap_2d(&maps.y, BF, 2, Y, T, m, m, PC_BM, PC_BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (ok && r16 > 0) {
    const __nv_bfloat16* z = static_cast<const __nv_bfloat16*>(h.zpre.p);
    ok = make_tmap_2d(&maps.u, BF, 2, h.U.p, m, h.r_pad, h.r_pad, 64, 128, SW) &&
         make_tmap_2d(&maps.zhi, BF, 2, z, T, r16, r16, 64, PC_BN, SW) &&
         make_tmap_2d(&maps.zlo, BF, 2, z + T * r16, T, r16, r16, 64, PC_BN, SW);
  }
  if (!ok) {
    set_message("tensor map encoding failed");
    return HSL_ERR_CUDA;
  }
  if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_prefill_csr), PC_SMEM))
    return cuda_fail(e, "CSR prefill smem attribute");
  const int64_t tiles = ((m + PC_BM - 1) / PC_BM) * ((T + PC_BN - 1) / PC_BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(tiles));
  cfg.blockDim = dim3(PC_THREADS);
  cfg.dynamicSmemBytes = PC_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = r16 > 0 ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cuda_fail(cudaLaunchKernelEx(&cfg, k_prefill_csr, maps, static_cast<const int32_t*>(h.prow.p),
                                      static_cast<const uint16_t*>(h.pcol.p),
                                      static_cast<const uint16_t*>(h.pval.p),
                                      static_cast<__nv_bfloat16*>(Y), int(m), int(n), int(T), r16,
                                      ystore, static_cast<uint32_t*>(h.err.p)),
                   "CSR prefill launch");
}

}  // namespace hsl
