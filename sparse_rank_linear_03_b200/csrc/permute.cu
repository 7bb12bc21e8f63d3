// Permutation for concentration: the ratio ρ, the reverse Cuthill–McKee order
// of a sparse pattern, the permuted copy of W and the permuted apply.
//
// "Hierarchical Sparse + Low-Rank Compression of LLMs", §Permutation and
// hierarchical alignment: rows and columns of W are reordered (RCM) so that the
// large entries gather near the diagonal, and the gain is measured by
//   ρ = Σ_{diagonal blocks} |W_ij| / Σ |W_ij|
// over the top-left and bottom-right blocks of the 2×2 partition (split at
// row ⌊m/2⌋ and column ⌊n/2⌋; an all-zero W has ρ = 0).  The order is kept so
// that the layer can be applied in the original order afterwards.
//
//   k_concentration  one pass over W (HBM-bound): CTAs take rows in a grid
//                    stride, threads 16-byte vectors of a row; |w| summed in
//                    fp64 per thread, a fixed tree per CTA, partials per CTA.
//   k_concentration_final  one CTA adds the partials in CTA order (the result
//                    does not depend on timing).
//   k_permute        W'[k][l] = W[row_order[k]][col_order[l]], a CTA per row
//                    of W' (bit copies).
//   k_gather_cols / k_scatter_rows  the permuted apply's x' = x[col_order]
//                    and y[row_order[k]] = y'[k].
//   rcm_order        host C++ (a one-off graph step, as the page describes):
//                    bipartite row–column graph of the pattern, start at the
//                    unvisited vertex of least degree (ties: lowest number),
//                    breadth first with neighbours by (degree, number), the
//                    whole order reversed.
#include <algorithm>
#include <cstring>
#include <numeric>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace hsl {
namespace {

constexpr int kRhoThreads = 256;

__device__ __forceinline__ double absval(uint16_t b) {
  return double(__uint_as_float(uint32_t(b & 0x7FFFu) << 16));
}
__device__ __forceinline__ double absval(uint32_t b) {
  return double(__uint_as_float(b & 0x7FFFFFFFu));
}

// partial[blockIdx][0] = Σ |w| over the diagonal blocks, [1] = Σ |w| over all
template <typename KT>
__global__ void __launch_bounds__(kRhoThreads) k_concentration(const KT* __restrict__ W, int64_t m,
                                                               int64_t n, int vec,
                                                               double* __restrict__ partial) {
  constexpr int PER = 16 / sizeof(KT);
  const int64_t mh = m / 2, nh = n / 2;
  double diag = 0.0, total = 0.0;
  for (int64_t i = blockIdx.x; i < m; i += gridDim.x) {
    const KT* row = W + i * n;
    const bool top = i < mh;
    double left = 0.0, right = 0.0;
    if (vec) {
      const int64_t nv = n / PER;
      for (int64_t v = threadIdx.x; v < nv; v += kRhoThreads) {
        const uint4 q = ld_stream16(row + v * PER);
        const KT* e = reinterpret_cast<const KT*>(&q);
        const int64_t j0 = v * PER;
#pragma unroll
        for (int t = 0; t < PER; ++t) {
          const double a = absval(e[t]);
          if (j0 + t < nh) left += a; else right += a;
        }
      }
    } else {
      for (int64_t j = threadIdx.x; j < n; j += kRhoThreads) {
        const double a = absval(row[j]);
        if (j < nh) left += a; else right += a;
      }
    }
    diag += top ? left : right;
    total += left + right;
  }
  __shared__ double sd[kRhoThreads], st[kRhoThreads];
  sd[threadIdx.x] = diag;
  st[threadIdx.x] = total;
  __syncthreads();
  for (int o = kRhoThreads / 2; o; o >>= 1) {
    if (threadIdx.x < o) {
      sd[threadIdx.x] += sd[threadIdx.x + o];
      st[threadIdx.x] += st[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    partial[2 * blockIdx.x] = sd[0];
    partial[2 * blockIdx.x + 1] = st[0];
  }
}

__global__ void k_concentration_final(const double* __restrict__ partial, int blocks,
                                      double* __restrict__ out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    double d = 0.0, t = 0.0;
    for (int b = 0; b < blocks; ++b) {
      d += partial[2 * b];
      t += partial[2 * b + 1];
    }
    out[0] = d;
    out[1] = t;
    out[2] = t > 0.0 ? d / t : 0.0;
  }
}

// A CTA per row of W': the source row is read whole (coalesced) into shared
// memory when it fits (staged), then gathered from there by the column order;
// wider rows gather straight from global memory.
template <typename KT>
__global__ void k_permute(const KT* __restrict__ W, int64_t m, int64_t n,
                          const int32_t* __restrict__ row_order, const int32_t* __restrict__ col_order,
                          KT* __restrict__ out, int staged) {
  extern __shared__ __align__(16) unsigned char prow_smem[];
  KT* rowbuf = reinterpret_cast<KT*>(prow_smem);
  for (int64_t k = blockIdx.x; k < m; k += gridDim.x) {
    const int32_t r = row_order[k];
    if (r < 0 || r >= m) continue;  // orders are checked on the host; never read out of bounds
    const KT* src = W + int64_t(r) * n;
    KT* dst = out + k * n;
    if (staged) {
      __syncthreads();
      for (int64_t l = threadIdx.x; l < n; l += blockDim.x) rowbuf[l] = src[l];
      __syncthreads();
      for (int64_t l = threadIdx.x; l < n; l += blockDim.x) {
        const int32_t c = col_order[l];
        if (c >= 0 && c < n) dst[l] = rowbuf[c];
      }
    } else {
      for (int64_t l = threadIdx.x; l < n; l += blockDim.x) {
        const int32_t c = col_order[l];
        if (c >= 0 && c < n) dst[l] = src[c];
      }
    }
  }
}

// x'[b][l] = x[b][col_order[l]]; y[b][row_order[k]] = y'[b][k]
template <typename KT>
__global__ void k_gather_cols(const KT* __restrict__ x, int64_t batch, int64_t n,
                              const int32_t* __restrict__ order, KT* __restrict__ out) {
  const int64_t total = batch * n;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t b = e / n, l = e - b * n;
    const int32_t o = order[l];
    out[e] = (o >= 0 && o < n) ? x[b * n + o] : KT(0);
  }
}
template <typename KT>
__global__ void k_scatter_rows(const KT* __restrict__ yp, int64_t batch, int64_t m,
                               const int32_t* __restrict__ order, KT* __restrict__ y) {
  const int64_t total = batch * m;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t b = e / m, k = e - b * m;
    const int32_t o = order[k];
    if (o >= 0 && o < m) y[b * m + o] = yp[e];
  }
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  return std::max(sms, 1);
}

}  // namespace

hsl_status concentration_run(const void* W, int64_t m, int64_t n, hsl_dtype dt, double* out_dev,
                             double* partial, int blocks, cudaStream_t s) {
  const int eb = dtype_bytes(dt);
  const int vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) && ((n * eb) % 16 == 0);
  if (dt == HSL_BF16)
    k_concentration<uint16_t><<<blocks, kRhoThreads, 0, s>>>(static_cast<const uint16_t*>(W), m, n,
                                                             vec, partial);
  else
    k_concentration<uint32_t><<<blocks, kRhoThreads, 0, s>>>(static_cast<const uint32_t*>(W), m, n,
                                                             vec, partial);
  note_launch();
  if (hsl_status e = cuda_fail(cudaGetLastError(), "concentration launch")) return e;
  k_concentration_final<<<1, 32, 0, s>>>(partial, blocks, out_dev);
  note_launch();
  return cuda_fail(cudaGetLastError(), "concentration final launch");
}

int concentration_blocks(int64_t m) {
  return int(std::max<int64_t>(1, std::min<int64_t>(m, int64_t(device_sms()) * 8)));
}

hsl_status permute_run(const void* W, int64_t m, int64_t n, hsl_dtype dt, const int32_t* row_order,
                       const int32_t* col_order, void* out, cudaStream_t s) {
  const unsigned grid = unsigned(std::max<int64_t>(1, std::min<int64_t>(m, int64_t(device_sms()) * 8)));
  const size_t row_bytes = size_t(n) * dtype_bytes(dt);
  const int staged = row_bytes <= 48 * 1024 ? 1 : 0;
  const size_t sm = staged ? row_bytes : 0;
  if (dt == HSL_BF16)
    k_permute<uint16_t><<<grid, 512, sm, s>>>(static_cast<const uint16_t*>(W), m, n, row_order,
                                             col_order, static_cast<uint16_t*>(out), staged);
  else
    k_permute<uint32_t><<<grid, 512, sm, s>>>(static_cast<const uint32_t*>(W), m, n, row_order,
                                             col_order, static_cast<uint32_t*>(out), staged);
  note_launch();
  return cuda_fail(cudaGetLastError(), "permute launch");
}

hsl_status gather_cols_run(const void* x, int64_t batch, int64_t n, hsl_dtype dt,
                           const int32_t* order, void* out, cudaStream_t s) {
  const int64_t total = batch * n;
  const unsigned grid = unsigned(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256,
                                                                       int64_t(device_sms()) * 8)));
  if (dt == HSL_BF16)
    k_gather_cols<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(x), batch, n, order,
                                                static_cast<uint16_t*>(out));
  else
    k_gather_cols<uint32_t><<<grid, 256, 0, s>>>(static_cast<const uint32_t*>(x), batch, n, order,
                                                static_cast<uint32_t*>(out));
  note_launch();
  return cuda_fail(cudaGetLastError(), "permuted apply gather launch");
}

hsl_status scatter_rows_run(const void* yp, int64_t batch, int64_t m, hsl_dtype dt,
                            const int32_t* order, void* y, cudaStream_t s) {
  const int64_t total = batch * m;
  const unsigned grid = unsigned(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256,
                                                                       int64_t(device_sms()) * 8)));
  if (dt == HSL_BF16)
    k_scatter_rows<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(yp), batch, m, order,
                                                 static_cast<uint16_t*>(y));
  else
    k_scatter_rows<uint32_t><<<grid, 256, 0, s>>>(static_cast<const uint32_t*>(yp), batch, m, order,
                                                 static_cast<uint32_t*>(y));
  note_launch();
  return cuda_fail(cudaGetLastError(), "permuted apply scatter launch");
}

// Reverse Cuthill–McKee on the bipartite row–column graph (host).
hsl_status rcm_order(int64_t m, int64_t n, const int32_t* row_ptr, const int32_t* col,
                     int32_t* row_order, int32_t* col_order) {
  const int64_t V = m + n;
  const int64_t nnz = row_ptr[m];
  // adjacency: rows → columns (the CSR itself), columns → rows (its transpose)
  std::vector<int64_t> cptr(size_t(n) + 1, 0);
  for (int64_t e = 0; e < nnz; ++e) {
    const int32_t j = col[e];
    if (j < 0 || j >= n) {
      set_message("column index outside [0, n) in the pattern");
      return HSL_ERR_INVALID_ARG;
    }
    ++cptr[size_t(j) + 1];
  }
  for (int64_t i = 0; i < m; ++i)
    if (row_ptr[i + 1] < row_ptr[i]) {
      set_message("row_ptr is not monotone");
      return HSL_ERR_INVALID_ARG;
    }
  for (int64_t j = 0; j < n; ++j) cptr[size_t(j) + 1] += cptr[size_t(j)];
  std::vector<int32_t> crow(size_t(std::max<int64_t>(nnz, 1)));
  {
    std::vector<int64_t> fill(cptr.begin(), cptr.end() - 1);
    for (int64_t i = 0; i < m; ++i)
      for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) crow[size_t(fill[size_t(col[e])]++)] = int32_t(i);
  }
  std::vector<int64_t> deg(static_cast<size_t>(V));
  for (int64_t i = 0; i < m; ++i) deg[size_t(i)] = row_ptr[i + 1] - row_ptr[i];
  for (int64_t j = 0; j < n; ++j) deg[size_t(m + j)] = cptr[size_t(j) + 1] - cptr[size_t(j)];
  auto less = [&](int64_t a, int64_t b) { return deg[size_t(a)] != deg[size_t(b)] ? deg[size_t(a)] < deg[size_t(b)] : a < b; };
  std::vector<int64_t> starts(static_cast<size_t>(V));
  std::iota(starts.begin(), starts.end(), int64_t(0));
  std::sort(starts.begin(), starts.end(), less);
  std::vector<char> visited(static_cast<size_t>(V), 0);
  std::vector<int64_t> order;
  order.reserve(size_t(V));
  std::vector<int64_t> fresh;
  for (int64_t st : starts) {
    if (visited[size_t(st)]) continue;
    visited[size_t(st)] = 1;
    size_t head = order.size();
    order.push_back(st);
    while (head < order.size()) {
      const int64_t v = order[head++];
      fresh.clear();
      if (v < m) {
        for (int64_t e = row_ptr[v]; e < row_ptr[v + 1]; ++e) {
          const int64_t u = m + col[e];
          if (!visited[size_t(u)]) {
            visited[size_t(u)] = 1;
            fresh.push_back(u);
          }
        }
      } else {
        const int64_t j = v - m;
        for (int64_t e = cptr[size_t(j)]; e < cptr[size_t(j) + 1]; ++e) {
          const int64_t u = crow[size_t(e)];
          if (!visited[size_t(u)]) {
            visited[size_t(u)] = 1;
            fresh.push_back(u);
          }
        }
      }
      std::sort(fresh.begin(), fresh.end(), less);
      order.insert(order.end(), fresh.begin(), fresh.end());
    }
  }
  std::reverse(order.begin(), order.end());
  int64_t ri = 0, ci = 0;
  for (int64_t v : order) {
    if (v < m) row_order[ri++] = int32_t(v);
    else col_order[ci++] = int32_t(v - m);
  }
  return HSL_OK;
}

}  // namespace hsl
