// hsl_split_topk_noalloc: the magnitude top-k split for callers that cannot
// allocate device memory.
//
// Some callers of this library are not allowed to call cudaMalloc: code that
// runs inside a serving runtime or plugin host that owns every byte of device
// memory and hands out only pre-planned buffers, code that must not trigger
// the device-wide synchronisation cudaMalloc/cudaFree can cause, or a caller
// that has no handle to keep workspace alive between calls.  This entry point
// takes the input and every output from the caller and keeps its own scratch
// (histogram, selection state, row ticket, look-back flags) in one file-scope
// __device__ array of fixed size, so it allocates nothing.
//
// Costs and rules that come with that:
//   * the array (kNoAllocBytes, about 2.2 MB) exists on every GPU that loads
//     libhsl, for the life of the process;
//   * all calls share it: calls that can overlap on the GPU (different
//     streams, or different host threads on one device) race and corrupt each
//     other's results.  Serialise them on one stream;
//   * its address is looked up once per device, with that device current, by
//     the first call made on it (cudaGetSymbolAddress); make that first call
//     before any stream capture;
//   * sizes beyond the array (m > kNoAllocMaxRows, n > 2^31 - 1, or m·n ≥ 2^31)
//     are refused;
//   * the status word is required: it is the only way a caller learns of a
//     NaN in W or of a device wait that gave up.
//
// The kernels are the ones the handle-based split uses (split_kernels.cuh);
// only the scratch pointers differ.
#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"
#include "split_kernels.cuh"

namespace hsl {
namespace {
constexpr int64_t kNoAllocMaxRows = 65536;
constexpr size_t kNoAllocHist = 32768 * sizeof(unsigned);
constexpr size_t kNoAllocState = 256;  // SelState at +0, row ticket at +64
// look-back flags: one per row (per-row emit) or per 32 KB tile of W, m·n < 2^31
constexpr int64_t kNoAllocFlags = std::max<int64_t>(kNoAllocMaxRows, (int64_t(4) << 31) / kTileBytesLB);
constexpr size_t kNoAllocBytes = kNoAllocHist + kNoAllocState + size_t(kNoAllocFlags) * 8;
}  // namespace
}  // namespace hsl

// The scratch.  In host code this name is only a stand-in for the device
// array: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[hsl::kNoAllocBytes];

namespace hsl {
namespace {

struct DeviceScratch {
  unsigned char* ptr = nullptr;
  int sms = 0;
};
constexpr int kMaxDevices = 64;
DeviceScratch g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Set-up for the current device, done once: device address of the array.
hsl_status scratch_for_current_device(DeviceScratch& out) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_message("device ordinal out of range for the static scratch table");
    return HSL_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceScratch& d = g_dev[dev];
  if (!d.ptr) {
    void* p = nullptr;
    if (cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch))
      return cuda_fail(e, "cudaGetSymbolAddress of the static split scratch");
    int sms = 0;
    if (cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))
      return cuda_fail(e, "multiprocessor count");
    d.sms = std::max(sms, 1);
    d.ptr = static_cast<unsigned char*>(p);
  }
  out = d;
  return HSL_OK;
}

template <typename KT, typename SB>
hsl_status run_noalloc(const KT* W, int64_t m, int64_t n, int64_t k, int32_t* row_ptr,
                       int32_t* col, SB* val, KT* R, uint32_t* err, const DeviceScratch& d,
                       cudaStream_t s) {
  unsigned* hist = reinterpret_cast<unsigned*>(d.ptr);
  SelState* st = reinterpret_cast<SelState*>(d.ptr + kNoAllocHist);
  unsigned* ticket = reinterpret_cast<unsigned*>(d.ptr + kNoAllocHist + 64);
  unsigned long long* flags =
      reinterpret_cast<unsigned long long*>(d.ptr + kNoAllocHist + kNoAllocState);
  const int64_t count = m * n;
  const bool vec_ok = (reinterpret_cast<uintptr_t>(W) % 16 == 0) &&
                      (R == nullptr || reinterpret_cast<uintptr_t>(R) % 16 == 0) &&
                      ((n * int64_t(sizeof(KT))) % 16 == 0);
  // selection state starts fresh on every call (the array keeps the last call's contents)
  k_sel_init<<<1, 1, 0, s>>>(st, k == 0 ? 0u : uint32_t(k), k == 0 ? 0xFFFFFFFFu : 0u);
  note_launch();
  const int passes = sizeof(KT) == 2 ? 1 : 3;
  const int bits[3] = {sizeof(KT) == 2 ? 15 : 11, 11, 9};
  const int shifts[3] = {sizeof(KT) == 2 ? 0 : 20, 9, 0};
  const uint32_t* skip = nullptr;  // no sampled bracket here: every pass runs
  for (int p = 0; p < passes; ++p) {
    if (k == 0 && p > 0) break;
    if (cudaError_t e = cudaMemsetAsync(hist, 0, kNoAllocHist, s)) return cuda_fail(e, "memset");
    const size_t smem = (size_t(1) << bits[p]) * sizeof(unsigned);
    if (bits[p] == 15) {
      auto kern = k_split_hist<KT, 15>;
      if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(kern), int(smem)))
        return cuda_fail(e, "split histogram smem attribute");
      kern<<<d.sms, 1024, smem, s>>>(W, count, st, shifts[p], hist, err, vec_ok ? 1 : 0, skip);
    } else if (bits[p] == 11) {
      k_split_hist<KT, 11><<<d.sms * 2, 1024, smem, s>>>(W, count, st, shifts[p], hist, err,
                                                          vec_ok ? 1 : 0, skip);
    } else {
      k_split_hist<KT, 9><<<d.sms * 2, 1024, smem, s>>>(W, count, st, shifts[p], hist, err,
                                                         vec_ok ? 1 : 0, skip);
    }
    note_launch();
    if (hsl_status e = cuda_fail(cudaGetLastError(), "split histogram launch")) return e;
    if (k > 0) {
      k_split_select<<<1, 1024, 0, s>>>(hist, 1 << bits[p], shifts[p], st, skip);
      note_launch();
      if (hsl_status e = cuda_fail(cudaGetLastError(), "split select launch")) return e;
    }
  }
  // the ticket and the look-back flags must start at zero
  if (cudaError_t e = cudaMemsetAsync(ticket, 0, 4, s)) return cuda_fail(e, "memset");
  const int64_t nflags = std::max<int64_t>(m, (count * int64_t(sizeof(KT)) + kTileBytesLB - 1) / kTileBytesLB);
  if (cudaError_t e = cudaMemsetAsync(flags, 0, size_t(nflags) * 8, s)) return cuda_fail(e, "memset");
  if (vec_ok) {
    constexpr int TE = kTileBytesLB / int(sizeof(KT));
    const int64_t ntiles = (count + TE - 1) / TE;
    const size_t smem = size_t(kStages) * kTileBytesLB;
    auto kern = k_split_emit_tile<KT, SB, kTileBytesLB>;
    if (cudaError_t e = allow_dyn_smem(reinterpret_cast<const void*>(kern), int(smem)))
      return cuda_fail(e, "split emit smem attribute");
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kTileThreads, smem);
    const int64_t grid = std::min<int64_t>(ntiles, int64_t(d.sms) * std::max(occ, 1));
    kern<<<unsigned(std::max<int64_t>(grid, 1)), kTileThreads, smem, s>>>(
        W, m, count, make_fastdiv(uint32_t(n)), ntiles, st, ticket, flags, row_ptr, col, val, R,
        k, err, nullptr, nullptr);
  } else {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_split_emit<KT, SB>, kEmitThreads, 0);
    const int64_t grid = std::min<int64_t>(m, int64_t(d.sms) * std::max(occ, 1));
    k_split_emit<KT, SB><<<unsigned(grid), kEmitThreads, 0, s>>>(
        W, m, n, st, ticket, flags, row_ptr, col, val, R, k, err, vec_ok ? 1 : 0);
  }
  note_launch();
  return cuda_fail(cudaGetLastError(), "split emit launch");
}

}  // namespace
}  // namespace hsl

using namespace hsl;

extern "C" hsl_status hsl_split_topk_noalloc(const void* W, int64_t m, int64_t n, hsl_dtype w_dtype,
                                             double frac, int32_t* row_ptr, int32_t* col, void* val,
                                             hsl_dtype val_dtype, void* residual,
                                             uint32_t* status, hsl_stream stream) {
  set_message("");
  if (!W || !row_ptr) {
    set_message("W/row_ptr is NULL");
    return HSL_ERR_INVALID_ARG;
  }
  if (w_dtype != HSL_F32 && w_dtype != HSL_BF16) {
    set_message("unknown W dtype");
    return HSL_ERR_INVALID_ARG;
  }
  if (val_dtype != HSL_F32 && val_dtype != HSL_BF16) {
    set_message("unknown value dtype");
    return HSL_ERR_INVALID_ARG;
  }
  if (std::isnan(frac)) {
    set_message("frac is NaN");
    return HSL_ERR_INVALID_ARG;
  }
  if (m < 1 || n < 1) {
    set_message("m and n must be >= 1");
    return HSL_ERR_INVALID_ARG;
  }
  if (!status) {
    set_message("status is NULL: the no-allocation split reports NaN input and device waits "
                "that gave up only through it");
    return HSL_ERR_INVALID_ARG;
  }
  // n is bounded before m·n is formed, so the product cannot overflow
  if (m > kNoAllocMaxRows || n > INT32_MAX || m * n >= (int64_t(1) << 31)) {
    set_message("hsl_split_topk_noalloc handles at most " + std::to_string(kNoAllocMaxRows) +
                " rows and m*n < 2^31 (its scratch is a fixed static array)");
    return HSL_ERR_UNSUPPORTED;
  }
  const int64_t total = m * n;
  const int64_t k = frac <= 0.0 ? 0 : frac >= 1.0 ? total : int64_t(std::floor(frac * double(total)));
  if (k > 0 && (!col || !val)) {
    set_message("col/val is NULL");
    return HSL_ERR_INVALID_ARG;
  }
  DeviceScratch d;
  if (hsl_status e = scratch_for_current_device(d)) return e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = cudaMemsetAsync(status, 0, 4, s)) return cuda_fail(e, "status clear");
  if (w_dtype == HSL_BF16) {
    const uint16_t* w = static_cast<const uint16_t*>(W);
    uint16_t* r = static_cast<uint16_t*>(residual);
    if (val_dtype == HSL_BF16)
      return run_noalloc<uint16_t, uint16_t>(w, m, n, k, row_ptr, col, static_cast<uint16_t*>(val),
                                             r, status, d, s);
    return run_noalloc<uint16_t, uint32_t>(w, m, n, k, row_ptr, col, static_cast<uint32_t*>(val), r,
                                           status, d, s);
  }
  const uint32_t* w = static_cast<const uint32_t*>(W);
  uint32_t* r = static_cast<uint32_t*>(residual);
  if (val_dtype == HSL_BF16)
    return run_noalloc<uint32_t, uint16_t>(w, m, n, k, row_ptr, col, static_cast<uint16_t*>(val), r,
                                           status, d, s);
  return run_noalloc<uint32_t, uint32_t>(w, m, n, k, row_ptr, col, static_cast<uint32_t*>(val), r,
                                         status, d, s);
}
