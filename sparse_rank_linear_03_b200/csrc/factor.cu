// Stage 2 on the GPU: randomized truncated SVD of the residual, R ≈ U Vᵀ.
//
// "Hierarchical Sparse + Low-Rank Compression of LLMs", §Two-stage hierarchical
// sparse + low-rank compression, Stage 2: the residual left by Stage 1 is
// factored into an m×r and an n×r matrix (1024×64 twice in the worked
// example); the implementation flow gives the factorisation an O(n³) cost.
// The factors are the truncated SVD of R with √σ on each side, computed by the
// randomized range finder of Halko, Martinsson and Tropp with a caller-given
// Gaussian test matrix Ω [n×k], k = r + oversampling:
//   Y = R Ω;  Q = orth(Y);  q times { Z = Rᵀ Q; Q = orth(R Z) };
//   Bᵀ = Rᵀ Q;  B Bᵀ = W Λ Wᵀ;  σ = √λ;  U = Q W_r √Σ_r,  V = Bᵀ W_r / √Σ_r.
//
// Kernels:
//   k_split_terms  an fp32 (or bf16) matrix as bf16 terms hi + mid + lo
//                  (hi = bf16(x), mid = bf16(x − hi), lo = bf16(x − hi − mid);
//                  each difference is exact in fp32), optionally transposed,
//                  into a zero-padded K-major array.  bf16 input is one term.
//   k_gemm_tc      C[M×N] = Σ_{a+b<3} A_a[M×K] · B_bᵀ (N ≤ 512): the tall
//                  products R·Ω, Rᵀ·Q, R·Z on tcgen05 (TMA, 128-byte swizzle,
//                  fp32 accumulators in TMEM, one or two N halves); the term
//                  pairs make every product exact and the sums fp32, so the
//                  product is fp32-accurate although the MMA takes bf16.
//                  K may be split over CTAs (partials added in split order).
//   k_gram         G = CᵀC in fp64 over row chunks (partials added in order).
//   k_chol_orth    one CTA: Cholesky of G with diagonal pivoting, stopped at
//                  the first negligible pivot, then T = Π R⁻¹ (fp64), so C·T
//                  is an orthonormal basis of span(C).
//   k_jacobi_coop  cyclic two-sided Jacobi in fp64 on a k×k symmetric matrix,
//                  a cooperative grid with one CTA per rotation pair of a
//                  round (circle method), grid barriers between the row and
//                  column passes; eigenvalues sorted descending with their
//                  vectors.  Bounded sweeps and bounded barriers.
//   k_scale_cols   T = W · diag(f(λ)) for the basis changes.
//   k_small_gemm   C[M×K] · T[K×N] (K, N ≤ 512) in fp32, written row-major
//                  (fp32 or the layer dtype) or as split bf16 terms transposed
//                  (the next tall product's B operand).
// orth(Y) = Y·Π R⁻¹ from the pivoted Cholesky factor of YᵀY, then once more
// on the result (Cholesky QR twice, for orthogonality); pivots below 1e-10 of
// the largest diagonal end the factor, their directions become zero columns,
// so rank-deficient Y is handled.  Only the final B Bᵀ needs eigenvectors
// (Jacobi).
#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace hsl {
namespace {

// ---- split into bf16 terms --------------------------------------------------------
// out[t][orow][ocol] (row stride ld_out, term stride term_stride) for the
// element in[row][col] (row stride ld_in); orow/ocol swapped when transposing.
template <typename TIn>
__global__ void k_split_terms(const TIn* __restrict__ in, int64_t rows, int64_t cols,
                              int64_t ld_in, int nterms, int transpose, uint16_t* __restrict__ out,
                              int64_t ld_out, int64_t term_stride) {
  __shared__ float tile[32][33];
  const int64_t r0 = int64_t(blockIdx.y) * 32, c0 = int64_t(blockIdx.x) * 32;
  for (int dy = threadIdx.y; dy < 32; dy += blockDim.y) {
    const int64_t r = r0 + dy, c = c0 + threadIdx.x;
    float v = 0.f;
    if (r < rows && c < cols) {
      if constexpr (sizeof(TIn) == 2)
        v = __uint_as_float(uint32_t(in[r * ld_in + c]) << 16);
      else
        v = in[r * ld_in + c];
    }
    tile[dy][threadIdx.x] = v;
  }
  __syncthreads();
  for (int dy = threadIdx.y; dy < 32; dy += blockDim.y) {
    // output element (orow, ocol): consecutive threads write consecutive ocol
    int64_t orow, ocol;
    float v;
    if (transpose) {
      orow = c0 + dy;
      ocol = r0 + threadIdx.x;
      v = tile[threadIdx.x][dy];
      if (orow >= cols || ocol >= rows) continue;
    } else {
      orow = r0 + dy;
      ocol = c0 + threadIdx.x;
      v = tile[dy][threadIdx.x];
      if (orow >= rows || ocol >= cols) continue;
    }
    float rest = v;
    for (int t = 0; t < nterms; ++t) {
      const __nv_bfloat16 h = __float2bfloat16_rn(rest);
      out[int64_t(t) * term_stride + orow * ld_out + ocol] = __bfloat16_as_ushort(h);
      rest = rest - __bfloat162float(h);
    }
  }
}

// ---- tall GEMM on tcgen05 -------------------------------------------------------------
constexpr int GT_THREADS = 192;
constexpr int GT_BK = 64;
constexpr int GT_A = 128 * 128;  // A tile: 128 rows × 64 bf16

struct GemmMaps {
  CUtensorMap a;  // A terms [nA·M][ldK]  box {64, 128}  SW128
  CUtensorMap b;  // B terms [nB·N][ldK]  box {64, BH}   SW128
};
struct GemmArgs {
  float* C;          // [M][N] (or partial [split][M][N])
  uint32_t* err;
  int M, N, BH, nh;  // BH rows per N half, nh ∈ {1, 2}
  int nA, nB;        // terms of A and B
  int nkb, splits;   // K-blocks, K splits
  int stages, stage_bytes;
};

__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                      volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (tc::mbar_wait(bar, parity, err)) return true;
  *abort_flag = 1;
  return false;
}

// the term pairs (a, b) with a + b < 3, a < nA, b < nB, in a fixed order
__device__ __forceinline__ int pair_count(int nA, int nB) {
  int c = 0;
  for (int a = 0; a < nA; ++a)
    for (int b = 0; b < nB; ++b)
      if (a + b < 3) ++c;
  return c;
}
__device__ __forceinline__ void pair_at(int idx, int nA, int nB, int& pa, int& pb) {
  for (int a = 0; a < nA; ++a)
    for (int b = 0; b < nB; ++b)
      if (a + b < 3) {
        if (idx == 0) {
          pa = a;
          pb = b;
          return;
        }
        --idx;
      }
  pa = pb = 0;
}

__global__ void __launch_bounds__(GT_THREADS, 1)
    k_gemm_tc(const __grid_constant__ GemmMaps maps, const GemmArgs g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int ST = g.stages, SB = g.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * SB);
  uint64_t* empty = full + ST;
  uint64_t* accf = empty + ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x / g.splits, sp = blockIdx.x % g.splits;
  const int kb0 = int(int64_t(sp) * g.nkb / g.splits), kb1 = int(int64_t(sp + 1) * g.nkb / g.splits);
  const int npair = pair_count(g.nA, g.nB);
  const int steps = (kb1 - kb0) * npair;
  const int b_bytes = g.BH * 128;
  const uint32_t ncols = g.nh == 2 ? 512u : (g.BH <= 32 ? 32u : g.BH <= 64 ? 64u : g.BH <= 128 ? 128u : 256u);

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accf, 1);
    tc::fence_mbar_init();
    tc::prefetch_tmap(&maps.a);
    tc::prefetch_tmap(&maps.b);
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
      int issued[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int st = 0; st < steps; ++st) {
        const int s = st % ST;
        const uint32_t ph = (st / ST) & 1;
        if (!gwait(&empty[s], ph ^ 1, g.err, abrt)) break;
        const int kb = kb0 + st / npair;
        int pa, pb;
        pair_at(st % npair, g.nA, g.nB, pa, pb);
        unsigned char* base = smem + s * SB;
        tc::mbar_expect_tx(&full[s], GT_A + g.nh * b_bytes);
        tc::tma_load_2d(base, &maps.a, kb * GT_BK, pa * g.M + mt * 128, &full[s]);
        for (int h = 0; h < g.nh; ++h)
          tc::tma_load_2d(base + GT_A + h * b_bytes, &maps.b, kb * GT_BK,
                          pb * (g.nh * g.BH) + h * g.BH, &full[s]);
        ++issued[s];
      }
      for (int s = 0; s < ST; ++s)
        if (issued[s]) tc::mbar_wait(&full[s], (issued[s] - 1) & 1, g.err);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, g.BH);
      for (int st = 0; st < steps; ++st) {
        const int s = st % ST;
        const uint32_t ph = (st / ST) & 1;
        if (!gwait(&full[s], ph, g.err, abrt)) break;
        tc::tc_fence_after();
        unsigned char* base = smem + s * SB;
        const uint64_t ad = tc::desc_sw128(base);
        for (int h = 0; h < g.nh; ++h) {
          const uint64_t bd = tc::desc_sw128(base + GT_A + h * b_bytes);
#pragma unroll
          for (int k = 0; k < GT_BK / 16; ++k)
            tc::mma_bf16(tmem + uint32_t(h * 256), tc::desc_advance(ad, k * 32),
                         tc::desc_advance(bd, k * 32), idesc, (st > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(accf);
    }
    __syncwarp();  // lanes 1-31 wait here for lane 0
  } else {
    // epilogue: TMEM lane = row of the tile
    const int q = warp & 3;
    const int row = (q << 5) | lane;
    const int i = mt * 128 + row;
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    float* C = g.C + (g.splits > 1 ? int64_t(sp) * g.M * g.N : 0);
    const bool ok = tc::mbar_wait(accf, 0, g.err) && !*abrt;
    if (ok && steps > 0) {
      tc::tc_fence_after();
      for (int h = 0; h < g.nh; ++h) {
        for (int c0 = 0; c0 < g.BH; c0 += 32) {
          float v[32];
          tc::tmem_ld32(tmem + lane_base + uint32_t(h * 256 + c0), v);
          if (i < g.M) {
            float* dst = C + int64_t(i) * g.N + h * g.BH + c0;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              if (h * g.BH + c0 + j < g.N)
                *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          }
        }
      }
    } else if (i < g.M) {
      // an empty K range (or a wait that gave up) contributes zeros
      for (int c = 0; c < g.N; c += 4)
        *reinterpret_cast<float4*>(C + int64_t(i) * g.N + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc::tc_fence_before();
  tc::cta_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, ncols);
  }
}

// out = Σ_s part[s] (fixed order)
template <typename T>
__global__ void k_sum_parts(const T* __restrict__ part, int splits, int64_t count, T* __restrict__ out) {
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < count;
       e += int64_t(gridDim.x) * blockDim.x) {
    T acc = part[e];
    for (int s = 1; s < splits; ++s) acc += part[int64_t(s) * count + e];
    out[e] = acc;
  }
}

// ---- Gram matrix in fp64 -------------------------------------------------------------
// partial[p][i][j] = Σ_{rows in chunk p} C[row][i]·C[row][j], C [M][N] fp32.
__global__ void __launch_bounds__(256) k_gram(const float* __restrict__ C, int64_t M, int N,
                                              int chunks, double* __restrict__ partial) {
  __shared__ float ta[32][33], tb[32][33];
  const int ti = blockIdx.x, tj = blockIdx.y, p = blockIdx.z;
  const int64_t r0 = int64_t(p) * M / chunks, r1 = int64_t(p + 1) * M / chunks;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 × 8
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int64_t rb = r0; rb < r1; rb += 32) {
    for (int dy = ty; dy < 32; dy += 8) {
      const int64_t r = rb + dy;
      const int ca = ti * 32 + tx, cb = tj * 32 + tx;
      ta[dy][tx] = (r < r1 && ca < N) ? C[r * N + ca] : 0.f;
      tb[dy][tx] = (r < r1 && cb < N) ? C[r * N + cb] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int rr = 0; rr < 32; ++rr) {
      const double b = tb[rr][tx];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] += double(ta[rr][ty + 8 * u]) * b;
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = ti * 32 + ty + 8 * u, j = tj * 32 + tx;
    if (i < N && j < N) partial[(int64_t(p) * N + i) * N + j] = acc[u];
  }
}

// ---- orthonormal basis by pivoted Cholesky of the Gram matrix (one CTA) -----------------
// G = CᵀC [k][k] fp64.  Diagonal pivoting (largest remaining pivot first, ties to
// the lower position) gives Πᵀ G Π = RᵀR with R upper triangular; the
// factorisation stops at the first pivot at or below thr_rel · max diag(G) (the
// columns of C past it are, to rounding, combinations of the earlier ones).
// Then T = Π R⁻¹ on the kept rank (zero columns after it), so C·T has
// orthonormal columns spanning span(C).  R is kept column-major (Rc[i][t] =
// R[t][i]) so every dot product reads contiguous memory; Ri likewise for R⁻¹.
constexpr int CT = 1024;
constexpr int kMaxK = 512;
__global__ void __launch_bounds__(CT) k_chol_orth(const double* __restrict__ G, int k, double thr_rel,
                                                  double* __restrict__ Rc, double* __restrict__ Ri,
                                                  float* __restrict__ T) {
  __shared__ double d[kMaxK];
  __shared__ int perm[kMaxK];
  __shared__ double rv[CT / 32];
  __shared__ int ri[CT / 32];
  __shared__ int piv;
  __shared__ double pval, dmax0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = CT / 32;
  for (int i = tid; i < k; i += CT) {
    d[i] = G[int64_t(i) * k + i];
    perm[i] = i;
  }
  for (int e = tid; e < k * k; e += CT) {
    Rc[e] = 0.0;
    Ri[e] = 0.0;
  }
  __syncthreads();
  // (value, position) maximum over positions [j0, k): ties to the lower position
  auto argmax = [&](int j0) {
    double bv = -1.0;
    int bi = k;
    for (int i = j0 + tid; i < k; i += CT)
      if (d[i] > bv) { bv = d[i]; bi = i; }
    for (int o = 16; o; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) { rv[warp] = bv; ri[warp] = bi; }
    __syncthreads();
    if (tid == 0) {
      double v = rv[0];
      int p = ri[0];
      for (int w = 1; w < NW; ++w)
        if (rv[w] > v || (rv[w] == v && ri[w] < p)) { v = rv[w]; p = ri[w]; }
      piv = p;
      pval = v;
    }
    __syncthreads();
  };
  argmax(0);
  if (tid == 0) dmax0 = pval > 0.0 ? pval : 0.0;
  __syncthreads();
  int rank = k;
  for (int j = 0; j < k; ++j) {
    if (j > 0) argmax(j);
    const int p = piv;
    const double dp = pval;
    if (p >= k || !(dp > thr_rel * dmax0) || !(dp > 0.0)) {  // uniform: all read the same values
      rank = j;
      break;
    }
    if (p != j) {
      for (int t = tid; t < j; t += CT) {
        const double a = Rc[int64_t(j) * k + t];
        Rc[int64_t(j) * k + t] = Rc[int64_t(p) * k + t];
        Rc[int64_t(p) * k + t] = a;
      }
      if (tid == 0) {
        const double dt = d[j];
        d[j] = d[p];
        d[p] = dt;
        const int pt = perm[j];
        perm[j] = perm[p];
        perm[p] = pt;
      }
    }
    __syncthreads();
    const double rjj = sqrt(d[j]);
    const int gj = perm[j];
    // row j of R at the positions after j: a warp per position, fixed-order sums
    for (int i = j + 1 + warp; i < k; i += NW) {
      double s = 0.0;
      for (int t = lane; t < j; t += 32) s = fma(Rc[int64_t(j) * k + t], Rc[int64_t(i) * k + t], s);
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) {
        const double v = (G[int64_t(gj) * k + perm[i]] - s) / rjj;
        Rc[int64_t(i) * k + j] = v;
        d[i] -= v * v;
      }
    }
    if (tid == 0) Rc[int64_t(j) * k + j] = rjj;
    __syncthreads();
  }
  // R⁻¹ on the kept rank, a warp per column c (back substitution, bottom up):
  // Ri[c][i] = −(Σ_{l=i+1..c} R[i][l]·Ri[c][l]) / R[i][i],  Ri[c][c] = 1 / R[c][c]
  for (int c = warp; c < rank; c += NW) {
    if (lane == 0) Ri[int64_t(c) * k + c] = 1.0 / Rc[int64_t(c) * k + c];
    __syncwarp();
    for (int i = c - 1; i >= 0; --i) {
      double s = 0.0;
      for (int l = i + 1 + lane; l <= c; l += 32)
        s = fma(Rc[int64_t(l) * k + i], Ri[int64_t(c) * k + l], s);
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) Ri[int64_t(c) * k + i] = -s / Rc[int64_t(i) * k + i];
      __syncwarp();
    }
  }
  __syncthreads();
  // T[perm[i]][c] = R⁻¹[i][c] for c < rank (upper triangle), zero elsewhere
  for (int e = tid; e < k * k; e += CT) {
    const int i = e / k, c = e % k;
    T[int64_t(perm[i]) * k + c] = (c < rank && i <= c) ? float(Ri[int64_t(c) * k + i]) : 0.f;
  }
}

// ---- symmetric eigensolver (cooperative grid, one CTA per rotation pair) -------------------
// Cyclic two-sided Jacobi in fp64 on A [k][k] (overwritten), V [k][k] work;
// eigenvalues sorted descending into evals [k], their vectors into the
// columns of vecs [k][k].  A round of the circle method pairs every index
// with one other (a dummy when k is odd): CTA b owns pair b, computes its
// rotation from the round's A, rotates rows p and q, and after a grid barrier
// columns p and q of A and V.  Disjoint pairs touch disjoint rows (columns),
// so the order of the updates inside a pass does not matter and the result is
// the same on every run.  A rotation is skipped when |a_pq| is negligible
// against √|a_pp·a_qq| (relative 1e-16) or against the largest diagonal entry
// (relative 1e-18); the sweeps stop after one with no rotation (at most
// max_sweeps).  The grid barrier is a counter and a generation word in `sync`
// (zeroed by the host before each launch); a wait that runs out of polls sets the abort word
// and kErrTimeout, and from then on every barrier returns at once, so the
// kernel still ends.
constexpr int JC = 256;
// sync: [0] arrivals, [1] generation, [2] abort, [3] [4] sweep flags
__device__ __forceinline__ void grid_sync(unsigned* sync, unsigned nb, uint32_t* err) {
  __syncthreads();
  if (threadIdx.x == 0 && atomicAdd(&sync[2], 0u) == 0u) {
    const unsigned g = atomicAdd(&sync[1], 0u);
    __threadfence();
    if (atomicAdd(&sync[0], 1u) == nb - 1) {
      atomicExch(&sync[0], 0u);
      __threadfence();
      atomicAdd(&sync[1], 1u);
    } else {
      long long i = 0;
      while (atomicAdd(&sync[1], 0u) == g && atomicAdd(&sync[2], 0u) == 0u) {
        if (++i > kSpinLimit) {
          atomicExch(&sync[2], 1u);
          set_error(err, kErrTimeout);
          break;
        }
      }
    }
    __threadfence();
  }
  __syncthreads();
}

__global__ void __launch_bounds__(JC) k_jacobi_coop(double* __restrict__ A, double* __restrict__ V, int k,
                                                    int max_sweeps, double* __restrict__ evals,
                                                    double* __restrict__ vecs, unsigned* sync,
                                                    uint32_t* err) {
  __shared__ double cs_s, sn_s, red[JC / 32];
  __shared__ int p_s, q_s, cnt_s;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned G = gridDim.x;
  const int K = k + (k & 1);
  for (int64_t e = int64_t(b) * JC + tid; e < int64_t(k) * k; e += int64_t(G) * JC)
    V[e] = (e / k == e % k) ? 1.0 : 0.0;
  // scale of the absolute skip test: the largest |diagonal entry| (same in every CTA)
  double dm = 0.0;
  for (int i = tid; i < k; i += JC) dm = fmax(dm, fabs(A[int64_t(i) * k + i]));
  for (int o = 16; o; o >>= 1) dm = fmax(dm, __shfl_xor_sync(0xffffffffu, dm, o));
  if (lane == 0) red[warp] = dm;
  __syncthreads();
  double dmax = 0.0;
  for (int w = 0; w < JC / 32; ++w) dmax = fmax(dmax, red[w]);
  const double abs_tol = 1e-18 * dmax;
  grid_sync(sync, G, err);
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    bool rotated = false;
    for (int round = 0; round < K - 1; ++round) {
      if (tid == 0) {
        auto player = [&](int j) { return 1 + (j + round) % (K - 1); };
        int p = b == 0 ? 0 : player(b), q = b == 0 ? player(0) : player(K - 1 - b);
        if (p > q) { const int t = p; p = q; q = t; }
        double c = 1.0, sn = 0.0;
        if (q < k) {
          const double apq = A[int64_t(p) * k + q];
          const double app = A[int64_t(p) * k + p], aqq = A[int64_t(q) * k + q];
          if (fabs(apq) > abs_tol && fabs(apq) > 1e-16 * sqrt(fabs(app * aqq))) {
            const double tau = (aqq - app) / (2.0 * apq);
            const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
            c = 1.0 / sqrt(1.0 + t * t);
            sn = t * c;
            rotated = true;
          }
        }
        p_s = p;
        q_s = q;
        cs_s = c;
        sn_s = sn;
      }
      __syncthreads();
      const int p = p_s, q = q_s;
      const double c = cs_s, sn = sn_s;
      if (sn != 0.0)  // rows p, q: (p, q) ← (c·row_p − s·row_q, s·row_p + c·row_q)
        for (int j = tid; j < k; j += JC) {
          const double ap = A[int64_t(p) * k + j], aq = A[int64_t(q) * k + j];
          A[int64_t(p) * k + j] = c * ap - sn * aq;
          A[int64_t(q) * k + j] = sn * ap + c * aq;
        }
      grid_sync(sync, G, err);
      if (sn != 0.0)  // columns p, q of A and of V
        for (int j = tid; j < k; j += JC) {
          const double ap = A[int64_t(j) * k + p], aq = A[int64_t(j) * k + q];
          A[int64_t(j) * k + p] = c * ap - sn * aq;
          A[int64_t(j) * k + q] = sn * ap + c * aq;
          const double vp = V[int64_t(j) * k + p], vq = V[int64_t(j) * k + q];
          V[int64_t(j) * k + p] = c * vp - sn * vq;
          V[int64_t(j) * k + q] = sn * vp + c * vq;
        }
      grid_sync(sync, G, err);
    }
    // a sweep without any rotation ends the iteration (flags alternate by sweep)
    if (tid == 0 && rotated) atomicOr(&sync[3 + (sweep & 1)], 1u);
    grid_sync(sync, G, err);
    const bool stop = atomicAdd(&sync[3 + (sweep & 1)], 0u) == 0u;
    // the other flag was last read before this sweep's barriers: clear it for the next sweep
    if (tid == 0 && b == 0) atomicExch(&sync[3 + ((sweep + 1) & 1)], 0u);
    grid_sync(sync, G, err);
    if (stop) break;
  }
  // sort by descending eigenvalue (rank = entries ahead; ties by index); CTA b
  // places the columns i ≡ b (mod G)
  for (int i = b; i < k; i += G) {
    const double li = A[int64_t(i) * k + i];
    if (tid == 0) cnt_s = 0;
    __syncthreads();
    int ahead = 0;
    for (int j = tid; j < k; j += JC) {
      const double lj = A[int64_t(j) * k + j];
      if (lj > li || (lj == li && j < i)) ++ahead;
    }
    atomicAdd(&cnt_s, ahead);
    __syncthreads();
    const int rank = cnt_s;
    if (tid == 0) evals[rank] = li;
    for (int r = tid; r < k; r += JC) vecs[int64_t(r) * k + rank] = V[int64_t(r) * k + i];
    __syncthreads();
  }
}

// T[i][j] = W[i][j]·f(λ_j) for j < ncols (row stride ld_t), with
// mode 0: f = λ^{-1/2}, 1: f = λ^{1/4} (√σ), 2: f = λ^{-1/4} (1/√σ); an
// eigenvalue at or below thr_rel·λ_max (λ_max = lam[0]) drops its direction (f = 0).
__global__ void k_scale_cols(const double* __restrict__ W, const double* __restrict__ lam, int k,
                             int ncols, int ld_t, int mode, double thr_rel, float* __restrict__ T) {
  const double thr = thr_rel * fmax(lam[0], 0.0);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < k * ld_t; e += gridDim.x * blockDim.x) {
    const int i = e / ld_t, j = e % ld_t;
    double f = 0.0;
    if (j < ncols) {
      const double l = lam[j];
      if (mode == 0) f = l > thr ? 1.0 / sqrt(l) : 0.0;
      else if (mode == 1) f = l > thr ? sqrt(sqrt(l)) : 0.0;
      else f = l > thr ? 1.0 / sqrt(sqrt(l)) : 0.0;
    }
    T[e] = float(double(W[int64_t(i) * k + (j < k ? j : 0)]) * f);
  }
}

__global__ void k_sigma(const double* __restrict__ lam, int r, double thr_rel, float* __restrict__ sigma) {
  const double thr = thr_rel * fmax(lam[0], 0.0);
  for (int j = threadIdx.x; j < r; j += blockDim.x) sigma[j] = lam[j] > thr ? float(sqrt(lam[j])) : 0.f;
}

// ---- small GEMM: out = C[M][K]·T[K][N] (K, N ≤ 512) -------------------------------------
// mode 0: fp32 row-major out (row stride ld_out); mode 1: bf16 row-major;
// mode 2: 3 bf16 terms transposed: out[t][col][row] (row stride ld_out, term stride tstride)
constexpr int SG = 64;
__global__ void __launch_bounds__(256) k_small_gemm(const float* __restrict__ C, int64_t M, int K,
                                                    int ldc, const float* __restrict__ T, int N,
                                                    int ldt, int mode, void* __restrict__ out,
                                                    int64_t ld_out, int64_t tstride) {
  __shared__ float cs[32][SG + 1];  // [k][row]
  __shared__ float ts[32][SG + 1];  // [k][col]
  const int64_t row0 = int64_t(blockIdx.x) * SG;
  const int col0 = blockIdx.y * SG;
  const int tr = threadIdx.x & 15, tcn = threadIdx.x >> 4;  // 16 × 16 threads, 4×4 outputs
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int e = threadIdx.x; e < 32 * SG; e += 256) {
      const int kk = e & 31, rr = e >> 5;
      const int64_t r = row0 + rr;
      cs[kk][rr] = (r < M && k0 + kk < K) ? C[r * ldc + k0 + kk] : 0.f;
      const int cc = e & (SG - 1), k2 = e / SG;
      ts[k2][cc] = (k0 + k2 < K && col0 + cc < N) ? T[int64_t(k0 + k2) * ldt + col0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = cs[kk][tr + 16 * u];
        b[u] = ts[kk][tcn + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t r = row0 + tr + 16 * u;
    if (r >= M) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int c = col0 + tcn + 16 * v;
      if (c >= N) continue;
      const float x = acc[u][v];
      if (mode == 0) {
        static_cast<float*>(out)[r * ld_out + c] = x;
      } else if (mode == 1) {
        static_cast<uint16_t*>(out)[r * ld_out + c] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
      } else {
        float rest = x;
        for (int t = 0; t < 3; ++t) {
          const __nv_bfloat16 h = __float2bfloat16_rn(rest);
          static_cast<uint16_t*>(out)[t * tstride + int64_t(c) * ld_out + r] = __bfloat16_as_ushort(h);
          rest -= __bfloat162float(h);
        }
      }
    }
  }
}

// ---- host side ------------------------------------------------------------------------------

struct Work {
  DevBuf bufs[16];
  ~Work() {
    for (DevBuf& b : bufs) release(b);
  }
};

hsl_status launch_split(const void* in, bool in_bf16, int64_t rows, int64_t cols, int64_t ld_in,
                        int nterms, bool transpose, uint16_t* out, int64_t ld_out,
                        int64_t term_stride, cudaStream_t s) {
  dim3 grid(unsigned((cols + 31) / 32), unsigned((rows + 31) / 32));
  dim3 block(32, 8);
  if (in_bf16)
    k_split_terms<uint16_t><<<grid, block, 0, s>>>(static_cast<const uint16_t*>(in), rows, cols,
                                                   ld_in, nterms, transpose ? 1 : 0, out, ld_out,
                                                   term_stride);
  else
    k_split_terms<float><<<grid, block, 0, s>>>(static_cast<const float*>(in), rows, cols, ld_in,
                                                nterms, transpose ? 1 : 0, out, ld_out, term_stride);
  note_launch();
  return cuda_fail(cudaGetLastError(), "split terms launch");
}

// C[M][N] = Σ A_a · B_bᵀ; A terms [nA][M][ld] (term stride M·ld), B terms [nB][N][ld]
hsl_status gemm_tall(const uint16_t* A, int nA, int64_t M, const uint16_t* B, int nB, int N,
                     int64_t ld, float* C, float* part, int64_t part_cap, int num_sms,
                     uint32_t* err, cudaStream_t s) {
  const int nh = N > 256 ? 2 : 1;
  const int BH = nh == 2 ? N / 2 : N;
  const int nkb = int(ld / GT_BK);
  const int mtiles = int((M + 127) / 128);
  // split K when the tiles do not fill the SMs (each split keeps ≥ 8 K-blocks)
  int splits = 1;
  while (mtiles * (splits + 1) <= num_sms && nkb / (splits + 1) >= 8) ++splits;
  if (splits > 1 && int64_t(splits) * M * N > part_cap) splits = 1;
  const int stage_bytes = GT_A + nh * BH * 128;
  const int stages = std::min(6, (200 * 1024) / stage_bytes);
  const int smem = stages * stage_bytes + 1024 + 256;
  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_tmap_2d(&maps.a, BF, 2, A, int64_t(nA) * M, ld, ld, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&maps.b, BF, 2, B, int64_t(nB) * nh * BH, ld, ld, 64, BH,
                    CU_TENSOR_MAP_SWIZZLE_128B)) {
    set_message("tensor map encoding failed (factorisation)");
    return HSL_ERR_CUDA;
  }
  GemmArgs g;
  g.C = splits > 1 ? part : C;
  g.err = err;
  g.M = int(M);
  g.N = N;
  g.BH = BH;
  g.nh = nh;
  g.nA = nA;
  g.nB = nB;
  g.nkb = nkb;
  g.splits = splits;
  g.stages = stages;
  g.stage_bytes = stage_bytes;
  if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(k_gemm_tc), smem))
    return cuda_fail(e, "factor gemm smem attribute");
  k_gemm_tc<<<unsigned(mtiles * splits), GT_THREADS, smem, s>>>(maps, g);
  note_launch();
  if (hsl_status e = cuda_fail(cudaGetLastError(), "factor gemm launch")) return e;
  if (splits > 1) {
    const int64_t count = M * N;
    k_sum_parts<float><<<unsigned(std::min<int64_t>((count + 255) / 256, int64_t(num_sms) * 8)), 256, 0,
                         s>>>(part, splits, count, C);
    note_launch();
    return cuda_fail(cudaGetLastError(), "factor gemm reduce launch");
  }
  return HSL_OK;
}

hsl_status gram(const float* C, int64_t M, int N, double* part, int64_t part_cap, double* G,
                int num_sms, cudaStream_t s) {
  const int nt = (N + 31) / 32;
  int chunks = int(std::max<int64_t>(
      1, std::min<int64_t>({(M + 1023) / 1024, (int64_t(num_sms) * 4 + nt * nt - 1) / (nt * nt),
                            int64_t(64)})));
  while (chunks > 1 && int64_t(chunks) * N * N > part_cap) --chunks;
  k_gram<<<dim3(nt, nt, chunks), 256, 0, s>>>(C, M, N, chunks, part);
  note_launch();
  if (hsl_status e = cuda_fail(cudaGetLastError(), "gram launch")) return e;
  const int64_t count = int64_t(N) * N;
  k_sum_parts<double><<<unsigned((count + 255) / 256), 256, 0, s>>>(part, chunks, count, G);
  note_launch();
  return cuda_fail(cudaGetLastError(), "gram reduce launch");
}

hsl_status eig(double* G, int k, double* Vw, double* evals, double* vecs, unsigned* sync,
               uint32_t* err, cudaStream_t s) {
  if (cudaError_t e = cudaMemsetAsync(sync, 0, 8 * sizeof(unsigned), s))
    return cuda_fail(e, "eigensolver barrier reset");
  // one CTA per rotation pair, all resident at once (cooperative launch)
  const unsigned grid = unsigned((k + (k & 1)) / 2);
  int max_sweeps = 40;
  void* args[] = {&G, &Vw, &k, &max_sweeps, &evals, &vecs, &sync, &err};
  note_launch();
  return cuda_fail(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k_jacobi_coop), dim3(grid),
                                               dim3(JC), args, 0, s),
                   "eigensolver launch");
}

hsl_status small_gemm(const float* C, int64_t M, int K, int ldc, const float* T, int N, int ldt,
                      int mode, void* out, int64_t ld_out, int64_t tstride, cudaStream_t s) {
  dim3 grid(unsigned((M + SG - 1) / SG), unsigned((N + SG - 1) / SG));
  k_small_gemm<<<grid, 256, 0, s>>>(C, M, K, ldc, T, N, ldt, mode, out, ld_out, tstride);
  note_launch();
  return cuda_fail(cudaGetLastError(), "small gemm launch");
}

}  // namespace

hsl_status factor_randomized_run(const void* R, int64_t m, int64_t n, hsl_dtype dtype, int r, int k,
                                 const float* omega, int power_iters, void* U, void* V,
                                 hsl_dtype out_dtype, float* sigma, uint32_t* err, int num_sms,
                                 cudaStream_t s) {
  const int kp = k <= 256 ? int(round_up(k, 16)) : int(round_up(k, 32));
  const int64_t ldm = round_up(m, 64), ldn = round_up(n, 64);
  const int nA = dtype == HSL_BF16 ? 1 : 3;
  const int64_t mx = std::max(m, n);
  // an eigenvalue of a Gram matrix below this share of the largest is rounding
  // noise of a direction the data does not have (fp32 data, fp64 sums)
  const double thr_rel = 1e-10;
  Work w;
  enum { RA, RT, OT, QT, ZT, YB, QF, BT, PART, GP, G, VW, EV, EVEC, TT, SY, NB };
  const size_t sizes[NB] = {
      size_t(nA) * m * ldn * 2,          // R as K-major A terms
      size_t(nA) * n * ldm * 2,          // Rᵀ terms
      size_t(3) * kp * ldn * 2,          // Ωᵀ terms
      size_t(3) * kp * ldm * 2,          // Qᵀ terms
      size_t(3) * kp * ldn * 2,          // Zᵀ terms
      size_t(mx) * kp * 4,               // Y / Z, then the orthonormal basis (fp32)
      size_t(mx) * kp * 4,               // first-pass basis (fp32)
      size_t(n) * kp * 4,                // Bᵀ = Rᵀ Q
      size_t(4) * mx * kp * 4,           // GEMM split partials
      size_t(64) * kp * kp * 8,          // Gram partials
      size_t(kp) * kp * 8,               // Gram
      size_t(kp) * kp * 8,               // eigensolver work
      size_t(kp) * 8,                    // eigenvalues
      size_t(kp) * kp * 8,               // eigenvectors
      size_t(kp) * kp * 4,               // basis change T
      size_t(64),                        // eigensolver grid barrier
  };
  for (int b = 0; b < NB; ++b)
    if (hsl_status e = ensure(w.bufs[b], sizes[b], "factorisation workspace")) return e;
  auto U16 = [&](int b) { return static_cast<uint16_t*>(w.bufs[b].p); };
  auto F32 = [&](int b) { return static_cast<float*>(w.bufs[b].p); };
  auto F64 = [&](int b) { return static_cast<double*>(w.bufs[b].p); };
  for (int b : {RA, RT, OT, QT, ZT})
    if (cudaError_t e = cudaMemsetAsync(w.bufs[b].p, 0, sizes[b], s)) return cuda_fail(e, "memset");
  const bool rb = dtype == HSL_BF16;
  // R and Rᵀ as bf16 terms (one for bf16 R, three for fp32 R), Ωᵀ as three terms
  if (hsl_status e = launch_split(R, rb, m, n, n, nA, false, U16(RA), ldn, m * ldn, s)) return e;
  if (hsl_status e = launch_split(R, rb, m, n, n, nA, true, U16(RT), ldm, n * ldm, s)) return e;
  if (hsl_status e = launch_split(omega, false, n, k, k, 3, true, U16(OT), ldn, int64_t(kp) * ldn, s))
    return e;
  const int64_t part_cap = int64_t(sizes[PART] / 4), gp_cap = int64_t(sizes[GP] / 8);

  // Y [M][kp] in YB → orthonormal basis of its columns in YB (fp32) and as
  // transposed bf16 terms at `terms` (row stride ld): two passes of
  // basis = C · W Λ^{-1/2} from the Gram matrix CᵀC = W Λ Wᵀ.
  auto orth = [&](int64_t M, uint16_t* terms, int64_t ld) -> hsl_status {
    for (int pass = 0; pass < 2; ++pass) {
      const float* cur = pass == 0 ? F32(YB) : F32(QF);
      if (hsl_status e = gram(cur, M, kp, F64(GP), gp_cap, F64(G), num_sms, s)) return e;
      k_chol_orth<<<1, CT, 0, s>>>(F64(G), kp, thr_rel, F64(VW), F64(EVEC), F32(TT));
      note_launch();
      if (hsl_status e = cuda_fail(cudaGetLastError(), "pivoted Cholesky launch")) return e;
      if (pass == 0) {
        if (hsl_status e = small_gemm(cur, M, kp, kp, F32(TT), kp, kp, 0, F32(QF), kp, 0, s)) return e;
      } else {
        if (hsl_status e = small_gemm(cur, M, kp, kp, F32(TT), kp, kp, 0, F32(YB), kp, 0, s)) return e;
        if (hsl_status e = small_gemm(cur, M, kp, kp, F32(TT), kp, kp, 2, terms, ld, int64_t(kp) * ld, s))
          return e;
      }
    }
    return HSL_OK;
  };

  // Y = R Ω, Q = orth(Y)
  if (hsl_status e = gemm_tall(U16(RA), nA, m, U16(OT), 3, kp, ldn, F32(YB), F32(PART), part_cap,
                               num_sms, err, s))
    return e;
  if (hsl_status e = orth(m, U16(QT), ldm)) return e;
  for (int it = 0; it < power_iters; ++it) {
    // Z = Rᵀ Q; Y = R Z; Q = orth(Y)
    if (hsl_status e = gemm_tall(U16(RT), nA, n, U16(QT), 3, kp, ldm, F32(YB), F32(PART), part_cap,
                                 num_sms, err, s))
      return e;
    // Z = Rᵀ Q as three bf16 terms, transposed, for the next product: span(R Z)
    // is span(R Rᵀ Q) whether or not Z is orthonormalised first, and Q (whose
    // columns are orthonormal) keeps Z well scaled, so Z is used as it is
    if (hsl_status e = launch_split(F32(YB), false, n, kp, kp, 3, true, U16(ZT), ldn,
                                    int64_t(kp) * ldn, s))
      return e;
    if (hsl_status e = gemm_tall(U16(RA), nA, m, U16(ZT), 3, kp, ldn, F32(YB), F32(PART), part_cap,
                                 num_sms, err, s))
      return e;
    if (hsl_status e = orth(m, U16(QT), ldm)) return e;
  }
  // Bᵀ = Rᵀ Q; B Bᵀ = W Λ Wᵀ; σ = √λ; U = Q W_r √Σ_r; V = Bᵀ W_r / √Σ_r
  if (hsl_status e = gemm_tall(U16(RT), nA, n, U16(QT), 3, kp, ldm, F32(BT), F32(PART), part_cap,
                               num_sms, err, s))
    return e;
  if (hsl_status e = gram(F32(BT), n, kp, F64(GP), gp_cap, F64(G), num_sms, s)) return e;
  if (hsl_status e = eig(F64(G), kp, F64(VW), F64(EV), F64(EVEC),
                         static_cast<unsigned*>(w.bufs[SY].p), err, s))
    return e;
  // σ below thr_rel^{1/2} of σ_max: no direction (zero factor columns)
  k_sigma<<<1, 256, 0, s>>>(F64(EV), r, thr_rel, sigma);
  note_launch();
  if (hsl_status e = cuda_fail(cudaGetLastError(), "sigma launch")) return e;
  const int omode = out_dtype == HSL_BF16 ? 1 : 0;
  k_scale_cols<<<64, 256, 0, s>>>(F64(EVEC), F64(EV), kp, r, r, 1, thr_rel, F32(TT));
  note_launch();
  if (hsl_status e = cuda_fail(cudaGetLastError(), "basis change launch")) return e;
  if (hsl_status e = small_gemm(F32(YB), m, kp, kp, F32(TT), r, r, omode, U, r, 0, s)) return e;
  k_scale_cols<<<64, 256, 0, s>>>(F64(EVEC), F64(EV), kp, r, r, 2, thr_rel, F32(TT));
  note_launch();
  if (hsl_status e = cuda_fail(cudaGetLastError(), "basis change launch")) return e;
  if (hsl_status e = small_gemm(F32(BT), n, kp, kp, F32(TT), r, r, omode, V, r, 0, s)) return e;
  // the workspace is freed when `w` goes out of scope: wait for the kernels first
  return cuda_fail(cudaStreamSynchronize(s), "factorisation");
}

}  // namespace hsl
