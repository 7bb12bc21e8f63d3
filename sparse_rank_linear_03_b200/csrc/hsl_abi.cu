// C ABI of libhsl (declared in include/hsl.h): argument checks, ownership of
// device buffers, host-pointer staging and dispatch to the kernel launchers.
// No exception crosses this boundary and nothing aborts.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace hsl {

std::atomic<uint64_t> g_launches{0};
static thread_local std::string t_msg;

void set_message(const std::string& s) { t_msg = s; }

hsl_status cuda_fail(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return HSL_OK;
  set_message(std::string(what) + ": " + cudaGetErrorString(e));
  if (e == cudaErrorMemoryAllocation) return HSL_ERR_OOM;
  return HSL_ERR_CUDA;
}

namespace {
std::mutex g_attr_mu;
struct AttrEntry {
  int device;
  const void* func;
  int kind;  // 0 dynamic shared memory, 1 carveout
  int value;
};
std::vector<AttrEntry> g_attrs;  // a few dozen kernels at most

// The entry for (device, func, kind), or nullptr.
AttrEntry* find_attr(int device, const void* func, int kind) {
  for (AttrEntry& e : g_attrs)
    if (e.device == device && e.func == func && e.kind == kind) return &e;
  return nullptr;
}
}  // namespace

cudaError_t allow_dyn_smem(const void* func, int bytes) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return e;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  AttrEntry* a = find_attr(dev, func, 0);
  if (a && a->value >= bytes) return cudaSuccess;
  if (cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes))
    return e;
  if (a) a->value = bytes;
  else g_attrs.push_back({dev, func, 0, bytes});
  return cudaSuccess;
}

cudaError_t prefer_carveout(const void* func, int percent) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return e;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (AttrEntry* a = find_attr(dev, func, 1); a && a->value == percent) return cudaSuccess;
  if (cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, percent))
    return e;
  if (AttrEntry* a = find_attr(dev, func, 1)) a->value = percent;
  else g_attrs.push_back({dev, func, 1, percent});
  return cudaSuccess;
}

// HSL_FAULT_INJECT=alloc makes every device allocation fail; =zwait makes the
// batch-1 2:4 decode's wait for z give up (host-side failure testing; no
// device fault is involved).
bool fault_injected(const char* what) {
  const char* v = std::getenv("HSL_FAULT_INJECT");
  return v && std::strcmp(v, what) == 0;
}
static bool inject_alloc_failure() { return fault_injected("alloc"); }

hsl_status ensure(DevBuf& b, size_t bytes, const char* what) {
  if (bytes <= b.bytes && b.p) return HSL_OK;
  if (inject_alloc_failure()) {
    set_message(std::string("allocation of ") + what + " failed (HSL_FAULT_INJECT=alloc)");
    return HSL_ERR_OOM;
  }
  if (b.p) cudaFree(b.p);
  b.p = nullptr;
  b.bytes = 0;
  const size_t want = bytes ? bytes : 16;
  if (cudaError_t e = cudaMalloc(&b.p, want)) {
    b.p = nullptr;
    cudaGetLastError();
    set_message(std::string("allocation of ") + what + " (" + std::to_string(want) +
                " bytes) failed: " + cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? HSL_ERR_OOM : HSL_ERR_CUDA;
  }
  b.bytes = want;
  return HSL_OK;
}

void release(DevBuf& b) {
  if (b.p) cudaFree(b.p);
  b.p = nullptr;
  b.bytes = 0;
}

namespace {

hsl_status invalid(const std::string& why) {
  set_message(why);
  return HSL_ERR_INVALID_ARG;
}
hsl_status unsupported(const std::string& why) {
  set_message(why);
  return HSL_ERR_UNSUPPORTED;
}

bool is_host_pointer(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return true;  // unknown to CUDA: plain host memory
  }
  return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

// Makes the handle's device current for the duration of a call.
struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      cudaGetLastError();
      prev = -1;
      return;
    }
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// A device array of `len` int32 that must hold each of 0..len-1 once: copied to
// the host and checked there (the permutation calls are one-off set-up steps).
hsl_status check_order(const int32_t* order_dev, int64_t len, const char* what, cudaStream_t s) try {
  std::vector<int32_t> h(static_cast<size_t>(len));
  if (cudaError_t e = cudaMemcpyAsync(h.data(), order_dev, size_t(len) * 4, cudaMemcpyDefault, s))
    return cuda_fail(e, "order copy");
  if (cudaError_t e = cudaStreamSynchronize(s)) return cuda_fail(e, "order copy");
  std::vector<char> seen(static_cast<size_t>(len), 0);
  for (int32_t v : h) {
    if (v < 0 || v >= len || seen[size_t(v)]) {
      set_message(std::string(what) + " is not a permutation of 0.." + std::to_string(len - 1));
      return HSL_ERR_INVALID_ARG;
    }
    seen[size_t(v)] = 1;
  }
  return HSL_OK;
} catch (const std::bad_alloc&) {
  set_message("host allocation failed while checking an order");
  return HSL_ERR_OOM;
}

hsl_status ensure_err_word(Handle& h, cudaStream_t s) {
  if (h.err.p) return HSL_OK;
  if (hsl_status e = ensure(h.err, 256, "error word")) return e;
  return cuda_fail(cudaMemsetAsync(h.err.p, 0, 256, s), "error word init");
}

void free_all(Handle& h) {
  DevBuf* bufs[] = {&h.row_ptr, &h.col, &h.val, &h.nm_val, &h.nm_idx, &h.prow, &h.pcol,
                    &h.pval, &h.pmeta, &h.pmeta_tc, &h.U, &h.Vt, &h.z,
                    &h.err, &h.split_ws, &h.flags, &h.tiles, &h.xstage, &h.ystage, &h.zpre, &h.sk_part, &h.sk_cnt, &h.sk_z, &h.perm_row, &h.perm_col, &h.xperm, &h.yperm, &h.pbase, &h.d8_lens, &h.plan.probs,
                    &h.plan.prob_row0, &h.plan.cta_rows, &h.plan.xy_ptrs, &h.plan.zsync};
  for (DevBuf* b : bufs) release(*b);
}

}  // namespace
}  // namespace hsl

using namespace hsl;

struct hsl_group_s {
  std::vector<hsl_handle> members;
  ApplyPlan plan;
  int device = 0;
  int num_sms = 148;
};

extern "C" {

const char* hsl_status_str(hsl_status st) {
  switch (st) {
    case HSL_OK: return "ok";
    case HSL_ERR_INVALID_ARG: return "invalid argument";
    case HSL_ERR_UNSUPPORTED: return "unsupported";
    case HSL_ERR_NOT_READY: return "not ready";
    case HSL_ERR_OOM: return "out of device memory";
    case HSL_ERR_CUDA: return "CUDA error";
    case HSL_ERR_NAN_INPUT: return "NaN in input";
    case HSL_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* hsl_last_message(void) { return t_msg.c_str(); }

uint64_t hsl_launch_count(void) { return g_launches.load(); }

hsl_status hsl_create(int64_t m, int64_t n, int32_t r, hsl_format fmt, hsl_dtype dtype,
                      hsl_handle* out) {
  t_msg.clear();
  if (!out) return invalid("out is NULL");
  *out = nullptr;
  if (m < 1 || n < 1) return invalid("m and n must be >= 1");
  if (m > INT32_MAX || n > INT32_MAX || m * n >= (int64_t(1) << 31))
    return unsupported("m*n must be < 2^31");
  if (r < 0 || r > 256) return unsupported("rank must be in [0, 256]");
  if (fmt != HSL_FMT_CSR && fmt != HSL_FMT_NM24) return invalid("unknown format");
  if (dtype != HSL_F32 && dtype != HSL_BF16) return invalid("unknown dtype");
  if (fmt == HSL_FMT_NM24 && n % 4) return unsupported("2:4 needs n % 4 == 0");
  hsl_handle h = new (std::nothrow) hsl_handle_s;
  if (!h) return invalid("host allocation failed");
  Handle& H = h->h;
  H.m = m;
  H.n = n;
  H.r = r;
  H.r_pad = int32_t(round_up(r, 8));
  H.fmt = fmt;
  H.dtype = dtype;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  H.device = dev;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
    cudaGetLastError();
    sms = 148;
  }
  H.num_sms = sms;
  *out = h;
  return HSL_OK;
}

hsl_status hsl_destroy(hsl_handle h) {
  if (!h) return HSL_OK;
  {
    DeviceGuard g(h->h.device);
    if (h->h.err.p) cudaDeviceSynchronize();
    free_all(h->h);
    cudaGetLastError();
  }
  delete h;
  return HSL_OK;
}

hsl_status hsl_split_topk(hsl_handle h, const void* W, hsl_dtype w_dtype, double frac,
                          void* residual, hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  if (!W) return invalid("W is NULL");
  if (w_dtype != HSL_F32 && w_dtype != HSL_BF16) return invalid("unknown W dtype");
  if (std::isnan(frac)) return invalid("frac is NaN");
  Handle& H = h->h;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (H.fmt == HSL_FMT_NM24 && frac != 0.5)
    return unsupported("2:4 handles keep exactly half: frac must be 0.5");
  DeviceGuard g(H.device);
  if (hsl_status e = ensure_err_word(H, s)) return e;
  H.packed = false;
  if (H.fmt == HSL_FMT_NM24) {
    H.has_sparse = false;
    if (hsl_status e = split_24_run(H, W, w_dtype, residual, s)) return e;
    H.nnz = H.m * (H.n / 2);
    H.has_sparse = true;
    return HSL_OK;
  }
  const int64_t total = H.m * H.n;
  int64_t k;
  if (frac <= 0.0) k = 0;
  else if (frac >= 1.0) k = total;
  else k = int64_t(std::floor(frac * double(total)));
  H.has_sparse = false;
  if (hsl_status e = split_topk_run(H, W, w_dtype, k, residual, s)) return e;
  H.nnz = k;
  H.has_sparse = true;
  return HSL_OK;
}

hsl_status hsl_get_nnz(hsl_handle h, int64_t* nnz) {
  t_msg.clear();
  if (!h || !nnz) return invalid("NULL argument");
  *nnz = h->h.has_sparse ? h->h.nnz : 0;
  return HSL_OK;
}

hsl_status hsl_get_sparse(hsl_handle h, int32_t* row_ptr, int32_t* col, void* val, uint8_t* nm_idx,
                          hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (!H.has_sparse) {
    set_message("no sparse part yet (split or set first)");
    return HSL_ERR_NOT_READY;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  const size_t eb = size_t(dtype_bytes(H.dtype));
  if (H.fmt == HSL_FMT_CSR) {
    if (!row_ptr || (H.nnz && (!col || !val))) return invalid("row_ptr/col/val is NULL");
    if (cudaError_t e = cudaMemcpyAsync(row_ptr, H.row_ptr.p, size_t(H.m + 1) * 4,
                                        cudaMemcpyDeviceToDevice, s))
      return cuda_fail(e, "export row_ptr");
    if (H.nnz) {
      if (cudaError_t e = cudaMemcpyAsync(col, H.col.p, size_t(H.nnz) * 4, cudaMemcpyDeviceToDevice, s))
        return cuda_fail(e, "export col");
      if (cudaError_t e = cudaMemcpyAsync(val, H.val.p, size_t(H.nnz) * eb, cudaMemcpyDeviceToDevice, s))
        return cuda_fail(e, "export val");
    }
    return HSL_OK;
  }
  if (!val || !nm_idx) return invalid("val/nm_idx is NULL");
  if (cudaError_t e = cudaMemcpyAsync(val, H.nm_val.p, size_t(H.m) * (H.n / 2) * eb,
                                      cudaMemcpyDeviceToDevice, s))
    return cuda_fail(e, "export 2:4 values");
  return cuda_fail(cudaMemcpyAsync(nm_idx, H.nm_idx.p, size_t(H.m) * (H.n / 4),
                                   cudaMemcpyDeviceToDevice, s),
                   "export 2:4 indices");
}

hsl_status hsl_set_sparse_csr(hsl_handle h, int64_t nnz, const int32_t* row_ptr,
                              const int32_t* col, const void* val, hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (H.fmt != HSL_FMT_CSR) return invalid("handle is not CSR");
  if (nnz < 0 || nnz > H.m * H.n) return invalid("nnz out of range");
  if (!row_ptr || (nnz && (!col || !val))) return invalid("row_ptr/col/val is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  if (hsl_status e = ensure_err_word(H, s)) return e;
  const size_t eb = size_t(dtype_bytes(H.dtype));
  H.packed = false;
  H.has_sparse = false;
  if (hsl_status e = ensure(H.row_ptr, size_t(H.m + 1) * 4, "CSR row_ptr")) return e;
  if (hsl_status e = ensure(H.col, size_t(std::max<int64_t>(nnz, 1)) * 4, "CSR col")) return e;
  if (hsl_status e = ensure(H.val, size_t(std::max<int64_t>(nnz, 1)) * eb, "CSR val")) return e;
  if (cudaError_t e = cudaMemcpyAsync(H.row_ptr.p, row_ptr, size_t(H.m + 1) * 4,
                                      cudaMemcpyDefault, s))
    return cuda_fail(e, "import row_ptr");
  if (nnz) {
    if (cudaError_t e = cudaMemcpyAsync(H.col.p, col, size_t(nnz) * 4, cudaMemcpyDefault, s))
      return cuda_fail(e, "import col");
    if (cudaError_t e = cudaMemcpyAsync(H.val.p, val, size_t(nnz) * eb, cudaMemcpyDefault, s))
      return cuda_fail(e, "import val");
  }
  H.nnz = nnz;
  H.has_sparse = true;
  return HSL_OK;
}

hsl_status hsl_set_sparse_nm24(hsl_handle h, const void* val, const uint8_t* nm_idx,
                               hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (H.fmt != HSL_FMT_NM24) return invalid("handle is not 2:4");
  if (!val || !nm_idx) return invalid("val/nm_idx is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  if (hsl_status e = ensure_err_word(H, s)) return e;
  const size_t eb = size_t(dtype_bytes(H.dtype));
  const size_t half = size_t(H.m) * size_t(H.n / 2);
  H.packed = false;
  H.has_sparse = false;
  if (hsl_status e = ensure(H.nm_val, half * eb, "2:4 values")) return e;
  if (hsl_status e = ensure(H.nm_idx, size_t(H.m) * size_t(H.n / 4), "2:4 indices")) return e;
  if (cudaError_t e = cudaMemcpyAsync(H.nm_val.p, val, half * eb, cudaMemcpyDefault, s))
    return cuda_fail(e, "import 2:4 values");
  if (cudaError_t e = cudaMemcpyAsync(H.nm_idx.p, nm_idx, size_t(H.m) * size_t(H.n / 4),
                                      cudaMemcpyDefault, s))
    return cuda_fail(e, "import 2:4 indices");
  H.nnz = int64_t(half);
  H.has_sparse = true;
  return HSL_OK;
}

hsl_status hsl_pack(hsl_handle h, const void* U, const void* V, hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (H.r > 0 && (!U || !V)) return invalid("U/V is NULL");
  if (!H.has_sparse) {
    set_message("no sparse part yet (split or set first)");
    return HSL_ERR_NOT_READY;
  }
  if (H.fmt == HSL_FMT_CSR && (H.index_bits == 16 || H.index_bits == 8) && H.n >= 65535)
    return unsupported("8- and 16-bit packed CSR columns need n < 65535");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  H.packed = false;
  if (hsl_status e = ensure_err_word(H, s)) return e;
  if (hsl_status e = pack_sparse_run(H, s)) return e;
  if (hsl_status e = pack_factors_run(H, U, V, s)) return e;
  Handle* one = &H;
  if (hsl_status e = plan_build(H.plan, &one, 1, s)) return e;
  H.csr_ascending = false;
  if (H.fmt == HSL_FMT_CSR) {  // the plan upload has synchronised s
    uint32_t unordered = 1;
    if (cudaError_t e = cudaMemcpy(&unordered, static_cast<uint32_t*>(H.err.p) + 1, 4,
                                   cudaMemcpyDeviceToHost))
      return cuda_fail(e, "column order flag read");
    H.csr_ascending = unordered == 0 && H.idx_bits == 16;
  }
  H.packed = true;
  return HSL_OK;
}

hsl_status hsl_set_index_bits(hsl_handle h, int32_t bits) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (bits != 0 && bits != 8 && bits != 16 && bits != 32) return invalid("bits must be 0, 8, 16 or 32");
  if (H.fmt != HSL_FMT_CSR) return unsupported("column widths apply to CSR handles");
  if ((bits == 8 || bits == 16) && H.n >= 65535)
    return unsupported("8- and 16-bit packed CSR columns need n < 65535");
  H.index_bits = bits;
  H.packed = false;
  return HSL_OK;
}

hsl_status hsl_apply(hsl_handle h, const void* X, void* Y, int64_t batch, hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  if (batch < 0) return invalid("batch < 0");
  if (batch == 0) return HSL_OK;
  if (!X || !Y) return invalid("X/Y is NULL");
  Handle& H = h->h;
  if (!H.packed) {
    set_message("hsl_pack has not been called since the last split/set");
    return HSL_ERR_NOT_READY;
  }
  if (batch > INT32_MAX / 2) return unsupported("batch too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  const size_t eb = size_t(dtype_bytes(H.dtype));
  const bool xh = is_host_pointer(X), yh = is_host_pointer(Y);
  const void* Xd = X;
  void* Yd = Y;
  if (xh) {
    if (hsl_status e = ensure(H.xstage, size_t(batch) * H.n * eb, "X staging")) return e;
    if (cudaError_t e = cudaMemcpyAsync(H.xstage.p, X, size_t(batch) * H.n * eb,
                                        cudaMemcpyHostToDevice, s))
      return cuda_fail(e, "X host-to-device");
    Xd = H.xstage.p;
  }
  if (yh) {
    if (hsl_status e = ensure(H.ystage, size_t(batch) * H.m * eb, "Y staging")) return e;
    Yd = H.ystage.p;
  }
  // permuted layer: x' = x[col_order], y' = Ŵ' x', y[row_order] = y'
  void* Yout = Yd;
  if (H.permuted) {
    if (hsl_status e = ensure(H.xperm, size_t(batch) * H.n * eb, "permuted X")) return e;
    if (hsl_status e = ensure(H.yperm, size_t(batch) * H.m * eb, "permuted Y")) return e;
    if (hsl_status e = gather_cols_run(Xd, batch, H.n, H.dtype,
                                       static_cast<const int32_t*>(H.perm_col.p), H.xperm.p, s))
      return e;
    Xd = H.xperm.p;
    Yd = H.yperm.p;
  }
  if (batch >= kPrefillMinBatch && prefill_supported(H, Xd)) {
    if (hsl_status e = apply_prefill_run(H, Xd, Yd, batch, s)) return e;
  } else if (batch >= kPrefillMinBatch && prefill_csr_supported(H, Xd)) {
    if (hsl_status e = apply_prefill_csr_run(H, Xd, Yd, batch, s)) return e;
  } else if (splitk_supported(H, Xd, batch)) {
    if (hsl_status e = apply_splitk_run(H, Xd, Yd, batch, s)) return e;
  } else {
    if (hsl_status e = apply_decode_run(H.plan, Xd, Yd, nullptr, batch, H.num_sms, s)) return e;
  }
  if (H.permuted) {
    if (hsl_status e = scatter_rows_run(Yd, batch, H.m, H.dtype,
                                        static_cast<const int32_t*>(H.perm_row.p), Yout, s))
      return e;
    Yd = Yout;
  }
  if (yh)
    return cuda_fail(cudaMemcpyAsync(Y, Yd, size_t(batch) * H.m * eb, cudaMemcpyDeviceToHost, s),
                     "Y device-to-host");
  return HSL_OK;
}

hsl_status hsl_group_create(const hsl_handle* hs, int32_t count, hsl_group* out, hsl_stream stream) {
  t_msg.clear();
  if (!out) return invalid("out is NULL");
  *out = nullptr;
  if (!hs || count < 1) return invalid("need at least one handle");
  for (int i = 0; i < count; ++i) {
    if (!hs[i]) return invalid("NULL handle in group");
    if (!hs[i]->h.packed) {
      set_message("every handle of a group must be packed");
      return HSL_ERR_NOT_READY;
    }
    if (hs[i]->h.dtype != hs[0]->h.dtype || hs[i]->h.fmt != hs[0]->h.fmt)
      return unsupported("a group needs one format and one dtype");
    if (hs[i]->h.device != hs[0]->h.device) return unsupported("a group lives on one device");
    if (hs[i]->h.permuted) return unsupported("a group does not take permuted layers");
  }
  hsl_group g = new (std::nothrow) hsl_group_s;
  if (!g) return invalid("host allocation failed");
  g->members.assign(hs, hs + count);
  g->device = hs[0]->h.device;
  g->num_sms = hs[0]->h.num_sms;
  DeviceGuard dg(g->device);
  std::vector<Handle*> hh(count);
  for (int i = 0; i < count; ++i) hh[i] = &hs[i]->h;
  if (hsl_status e = plan_build(g->plan, hh.data(), count, static_cast<cudaStream_t>(stream))) {
    DevBuf* bufs[] = {&g->plan.probs, &g->plan.prob_row0, &g->plan.cta_rows, &g->plan.xy_ptrs,
                      &g->plan.zsync};
    for (DevBuf* b : bufs) release(*b);
    delete g;
    return e;
  }
  *out = g;
  return HSL_OK;
}

hsl_status hsl_group_apply(hsl_group g, const void* const* X, void* const* Y, int64_t batch,
                           hsl_stream stream) {
  t_msg.clear();
  if (!g) return invalid("group is NULL");
  if (!X || !Y) return invalid("X/Y table is NULL");
  if (batch < 0) return invalid("batch < 0");
  if (batch == 0) return HSL_OK;
  const int count = g->plan.count;
  for (int i = 0; i < count; ++i) {
    if (!X[i] || !Y[i]) return invalid("NULL X/Y in table");
    if (!g->members[i]->h.packed) {
      set_message("a member was split/set again after the group was created");
      return HSL_ERR_NOT_READY;
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard dg(g->device);
  // upload the pointer table only when it changed
  std::string tab(size_t(2 * count) * sizeof(void*), '\0');
  std::memcpy(&tab[0], X, size_t(count) * sizeof(void*));
  std::memcpy(&tab[size_t(count) * sizeof(void*)], Y, size_t(count) * sizeof(void*));
  if (tab != g->plan.host_xy) {
    if (hsl_status e = ensure(g->plan.xy_ptrs, tab.size(), "pointer table")) return e;
    if (cudaError_t e = cudaMemcpyAsync(g->plan.xy_ptrs.p, tab.data(), tab.size(),
                                        cudaMemcpyHostToDevice, s))
      return cuda_fail(e, "pointer table upload");
    g->plan.host_xy = tab;
  }
  return apply_decode_run(g->plan, nullptr, nullptr,
                          static_cast<const void* const*>(g->plan.xy_ptrs.p), batch, g->num_sms, s);
}

hsl_status hsl_group_destroy(hsl_group g) {
  if (!g) return HSL_OK;
  {
    DeviceGuard dg(g->device);
    if (g->plan.probs.p) cudaDeviceSynchronize();
    DevBuf* bufs[] = {&g->plan.probs, &g->plan.prob_row0, &g->plan.cta_rows, &g->plan.xy_ptrs,
                      &g->plan.zsync};
    for (DevBuf* b : bufs) release(*b);
    cudaGetLastError();
  }
  delete g;
  return HSL_OK;
}

hsl_status hsl_factor(hsl_handle h, const void* R, hsl_dtype r_dtype, const float* omega, int32_t k,
                      int32_t power_iters, void* U, void* V, float* sigma, hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (!R || !omega) return invalid("R/omega is NULL");
  if (r_dtype != HSL_F32 && r_dtype != HSL_BF16) return invalid("unknown R dtype");
  if (H.r == 0) return HSL_OK;
  if (!U || !V || !sigma) return invalid("U/V/sigma is NULL");
  if (k < H.r || k > 512) return unsupported("need r <= k <= 512 columns in omega");
  if (k > std::min(H.m, H.n)) return unsupported("need k <= min(m, n)");
  if (power_iters < 0 || power_iters > 64) return invalid("power_iters out of [0, 64]");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  if (hsl_status e = ensure_err_word(H, s)) return e;
  return factor_randomized_run(R, H.m, H.n, r_dtype, H.r, k, omega, power_iters, U, V, H.dtype,
                               sigma, static_cast<uint32_t*>(H.err.p), H.num_sms, s);
}

hsl_status hsl_concentration(const void* W, int64_t m, int64_t n, hsl_dtype dtype, double* rho,
                             hsl_stream stream) {
  t_msg.clear();
  if (!W || !rho) return invalid("W/rho is NULL");
  if (m < 1 || n < 1) return invalid("m and n must be >= 1");
  if (dtype != HSL_F32 && dtype != HSL_BF16) return invalid("unknown dtype");
  if (m > INT32_MAX || n > INT32_MAX || m * n >= (int64_t(1) << 40))
    return unsupported("matrix too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int blocks = concentration_blocks(m);
  // a small workspace per device, kept for later calls (calls on one device
  // are serialised by the lock: each waits for its result before returning)
  static std::mutex mu;
  static DevBuf ws[64];
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev)) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return unsupported("device ordinal out of range");
  std::lock_guard<std::mutex> lock(mu);
  if (hsl_status e = ensure(ws[dev], size_t(blocks) * 16 + 64, "concentration workspace")) return e;
  double* out = static_cast<double*>(ws[dev].p);
  hsl_status st = concentration_run(W, m, n, dtype, out, out + 8, blocks, s);
  double res[3] = {0.0, 0.0, 0.0};
  if (st == HSL_OK) {
    if (cudaError_t e = cudaMemcpyAsync(res, out, sizeof(res), cudaMemcpyDeviceToHost, s))
      st = cuda_fail(e, "concentration result");
    else if (cudaError_t e2 = cudaStreamSynchronize(s))
      st = cuda_fail(e2, "concentration result");
  }
  if (st == HSL_OK) *rho = res[2];
  return st;
}

hsl_status hsl_rcm_order(int64_t m, int64_t n, const int32_t* row_ptr, const int32_t* col,
                         int32_t* row_order, int32_t* col_order) {
  t_msg.clear();
  if (!row_ptr || !row_order || !col_order) return invalid("NULL argument");
  if (m < 1 || n < 1 || m > INT32_MAX || n > INT32_MAX) return invalid("m and n out of range");
  if (row_ptr[0] != 0) return invalid("row_ptr must start at 0");
  for (int64_t i = 0; i < m; ++i)
    if (row_ptr[i + 1] < row_ptr[i]) return invalid("row_ptr is not monotone");
  if (int64_t(row_ptr[m]) > m * n) return invalid("row_ptr[m] exceeds m*n");
  if (row_ptr[m] > 0 && !col) return invalid("col is NULL");
  try {
    return rcm_order(m, n, row_ptr, col, row_order, col_order);
  } catch (const std::bad_alloc&) {
    set_message("host allocation failed in the RCM order");
    return HSL_ERR_OOM;
  } catch (...) {
    set_message("RCM order failed");
    return HSL_ERR_INVALID_ARG;
  }
}

hsl_status hsl_permute(const void* W, int64_t m, int64_t n, hsl_dtype dtype,
                       const int32_t* row_order, const int32_t* col_order, void* out,
                       hsl_stream stream) {
  t_msg.clear();
  if (!W || !row_order || !col_order || !out) return invalid("NULL argument");
  if (m < 1 || n < 1 || m > INT32_MAX || n > INT32_MAX) return invalid("m and n out of range");
  if (dtype != HSL_F32 && dtype != HSL_BF16) return invalid("unknown dtype");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (hsl_status e = check_order(row_order, m, "row_order", s)) return e;
  if (hsl_status e = check_order(col_order, n, "col_order", s)) return e;
  return permute_run(W, m, n, dtype, row_order, col_order, out, s);
}

hsl_status hsl_set_permutation(hsl_handle h, const int32_t* row_order, const int32_t* col_order,
                               hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (!row_order && !col_order) {
    H.permuted = false;
    return HSL_OK;
  }
  if (!row_order || !col_order) return invalid("give both orders, or neither");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  if (hsl_status e = check_order(row_order, H.m, "row_order", s)) return e;
  if (hsl_status e = check_order(col_order, H.n, "col_order", s)) return e;
  if (hsl_status e = ensure(H.perm_row, size_t(H.m) * 4, "row order")) return e;
  if (hsl_status e = ensure(H.perm_col, size_t(H.n) * 4, "column order")) return e;
  if (cudaError_t e = cudaMemcpyAsync(H.perm_row.p, row_order, size_t(H.m) * 4, cudaMemcpyDefault, s))
    return cuda_fail(e, "row order copy");
  if (cudaError_t e = cudaMemcpyAsync(H.perm_col.p, col_order, size_t(H.n) * 4, cudaMemcpyDefault, s))
    return cuda_fail(e, "column order copy");
  H.permuted = true;
  return HSL_OK;
}

hsl_status hsl_check(hsl_handle h, hsl_stream stream) {
  t_msg.clear();
  if (!h) return invalid("handle is NULL");
  Handle& H = h->h;
  if (!H.err.p) return HSL_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceGuard g(H.device);
  if (cudaError_t e = cudaStreamSynchronize(s)) return cuda_fail(e, "stream synchronize");
  uint32_t word = 0;
  if (cudaError_t e = cudaMemcpy(&word, H.err.p, 4, cudaMemcpyDeviceToHost))
    return cuda_fail(e, "error word read");
  if (word == 0) return HSL_OK;
  if (cudaError_t e = cudaMemset(H.err.p, 0, 4)) return cuda_fail(e, "error word clear");
  if (word & kErrTimeout) {
    set_message("a bounded device wait gave up");
    return HSL_ERR_TIMEOUT;
  }
  if (word & kErrBadIndex) {
    set_message("a CSR column index was outside [0, n)");
    return HSL_ERR_INVALID_ARG;
  }
  set_message("W contains NaN");
  return HSL_ERR_NAN_INPUT;
}

}  // extern "C"
