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
}

extern "C" dig_status dig_gla_fwd_noalloc(const void* q, const void* k, const void* v, const float* z, int gate_heads,
                                          float inv_tau, void* o, const void* r, const float* gamma, float eps, void* y,
                                          int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                                          int scan_mode, int dtype, int out_dtype, unsigned int* device_status,
                                          void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DIG_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      // In host code g_scratch names a host-side stand-in; the kernel needs the
      // device address, resolved once per device with that device current.
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
      if (e != cudaSuccess || p == nullptr) return DIG_ERR_CUDA;
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
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
  if (cudaMemsetAsync(scratch, 0, kClearBytes, s) != cudaSuccess) return DIG_ERR_CUDA;
  const dig_status st = dig_gla_fwd(q, k, v, z, gate_heads, inv_tau, o, r, gamma, eps, y, B, H, L, d_k, d_v, grid_h,
                                    grid_w, scan_mode, dtype, out_dtype, scratch, kScratchBytes, stream);
  if (st != DIG_OK) return st;
  if (device_status != nullptr &&
      cudaMemcpyAsync(device_status, scratch, sizeof(unsigned int), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DIG_ERR_CUDA;
  return DIG_OK;
}
