// dig_noalloc.cu -- dig_gla_fwd_noalloc: the GLA forward for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: plug-ins hosted by a runtime that owns all
// device memory and forbids its extensions to allocate, and host programs that
// link only this library and have no device allocator of their own.  dig_gla_fwd
// needs a caller-allocated workspace; this entry point instead uses a scratch
// array built into the library (file-scope, one per GPU that loads the library,
// kept until the process exits) and allocates nothing.
#include <cstdio>
#include <mutex>

#include "../../include/dig.h"

namespace {

constexpr size_t kScratchBytes = 16u << 20;  // 16 MiB per device
constexpr size_t kClearBytes = 256;  // the header (status word)
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];  // device address of g_scratch, per device

}  // namespace

namespace dig {
void set_last_error(const char* msg);  // dig_api.cu
dig_status gla_fwd_check(const void* q, const void* k, const void* v, const float* z, int gate_heads, void* o,
                         const void* r, const float* gamma, void* y, int B, int H, int L, int d_k, int d_v,
                         int grid_h, int grid_w, int scan_mode, int dtype, int out_dtype, const void* workspace,
                         size_t workspace_bytes, bool* nothing_to_do);  // dig_api.cu
}

namespace {
dig_status cuda_fail(const char* step, cudaError_t e) {
  char msg[256];
  snprintf(msg, sizeof(msg), "dig_gla_fwd_noalloc: %s: %s", step, cudaGetErrorString(e));
  dig::set_last_error(msg);
  return DIG_ERR_CUDA;
}
}  // namespace

extern "C" dig_status dig_gla_fwd_noalloc(const void* q, const void* k, const void* v, const float* z, int gate_heads,
                                          float inv_tau, void* o, const void* r, const float* gamma, float eps, void* y,
                                          int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                                          int scan_mode, int dtype, int out_dtype, unsigned int* device_status,
                                          void* stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) {
    char msg[160];
    snprintf(msg, sizeof(msg), "dig_gla_fwd_noalloc: device %d is beyond the %d devices it keeps a scratch address for",
             dev, kMaxDevices);
    dig::set_last_error(msg);
    return DIG_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      // In host code g_scratch names a host-side stand-in; the kernel needs the
      // device address, resolved once per device with that device current.
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_scratch);
      if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress of the scratch array", e);
      if (p == nullptr) return cuda_fail("cudaGetSymbolAddress of the scratch array", cudaErrorInvalidSymbol);
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  // Every argument check of dig_gla_fwd runs before anything is enqueued.
  bool empty = false;
  dig_status st = dig::gla_fwd_check(q, k, v, z, gate_heads, o, r, gamma, y, B, H, L, d_k, d_v, grid_h, grid_w,
                                     scan_mode, dtype, out_dtype, scratch, ~size_t(0), &empty);
  if (st != DIG_OK) return st;
  const size_t need = dig_gla_workspace_bytes(B, H, gate_heads, L, d_k, d_v, 0);
  if (need > kScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "dig_gla_fwd_noalloc: this shape needs %zu bytes of workspace, the built-in scratch holds %zu; "
             "use dig_gla_fwd with a caller-allocated workspace",
             need, kScratchBytes);
    dig::set_last_error(msg);
    return DIG_ERR_WORKSPACE_TOO_SMALL;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word must start at zero on every call
  if ((e = cudaMemsetAsync(scratch, 0, kClearBytes, s)) != cudaSuccess) return cuda_fail("status clear", e);
  if (!empty) {
    st = dig_gla_fwd(q, k, v, z, gate_heads, inv_tau, o, r, gamma, eps, y, B, H, L, d_k, d_v, grid_h, grid_w,
                     scan_mode, dtype, out_dtype, scratch, kScratchBytes, stream);
    if (st != DIG_OK) return st;
  }
  if (device_status != nullptr &&
      (e = cudaMemcpyAsync(device_status, scratch, sizeof(unsigned int), cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return cuda_fail("status copy", e);
  return DIG_OK;
}
