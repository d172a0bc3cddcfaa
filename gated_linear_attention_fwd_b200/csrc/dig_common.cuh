// dig_common.cuh -- pieces shared by the DiG kernels: scan order, typed row
// loads/stores, workspace layout, device status word.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/dig.h"

namespace dig {

// Launches a kernel with programmatic stream serialization: it may be scheduled
// while the previous kernel of the stream is still running, and every kernel of
// this library waits (griddepcontrol.wait) before its first global memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Scan position t -> grid token index (DiG scanning directions).  Reversed
// modes visit the forward order backwards; column modes walk down each column.
__device__ __forceinline__ int scan_to_grid(int t, int L, int Hg, int Wg, int mode) {
  if (mode & 1) t = L - 1 - t;
  if (mode & 2) return (t % Hg) * Wg + t / Hg;
  return t;
}

// ------------------------------------------------------------------ element I/O
template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
};
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
};

// Load N consecutive elements (N % 4 == 0) starting at p into fp32 registers.
// bf16 rows use 8-byte loads (4 values), fp32 rows 16-byte loads.
template <int N>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float* out) {
  static_assert(N % 4 == 0, "row pieces are whole groups of 4");
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    uint2 u = __ldg(reinterpret_cast<const uint2*>(p + i));
    out[i + 0] = __uint_as_float(u.x << 16);
    out[i + 1] = __uint_as_float(u.x & 0xFFFF0000u);
    out[i + 2] = __uint_as_float(u.y << 16);
    out[i + 3] = __uint_as_float(u.y & 0xFFFF0000u);
  }
}
template <int N>
__device__ __forceinline__ void load_row(const float* p, float* out) {
  static_assert(N % 4 == 0, "row pieces are whole groups of 4");
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    float4 u = __ldg(reinterpret_cast<const float4*>(p + i));
    out[i + 0] = u.x;
    out[i + 1] = u.y;
    out[i + 2] = u.z;
    out[i + 3] = u.w;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&h);
}

// Store N consecutive values (N % 4 == 0).
template <int N>
__device__ __forceinline__ void store_row(__nv_bfloat16* p, const float* v) {
  static_assert(N % 4 == 0, "row pieces are whole groups of 4");
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    uint2 u;
    u.x = pack_bf16x2(v[i + 0], v[i + 1]);
    u.y = pack_bf16x2(v[i + 2], v[i + 3]);
    *reinterpret_cast<uint2*>(p + i) = u;
  }
}
template <int N>
__device__ __forceinline__ void store_row(float* p, const float* v) {
  static_assert(N % 4 == 0, "row pieces are whole groups of 4");
#pragma unroll
  for (int i = 0; i < N; i += 4) *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}

// log(sigmoid(x)) without overflow: min(x, 0) - log1p(exp(-|x|)).
__device__ __forceinline__ float log_sigmoid(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }

// ------------------------------------------------------------------ workspace
// Header (256 bytes) followed by the gate factors and per-chunk records.
struct WsHeader {
  uint32_t status;  // first device-side condition (0 = none)
  uint32_t pad[63];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code) { atomicCAS(status, 0u, code); }

// Bound of every wait on the tensor core's completion barriers: far beyond any
// legitimate wait; on expiry the kernel records DIG_ERR_DEVICE_TIMEOUT.
constexpr uint64_t kSpinLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

}  // namespace dig
