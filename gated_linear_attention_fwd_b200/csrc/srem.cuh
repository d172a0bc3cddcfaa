// srem.cuh -- pieces shared by the SREM conv kernels (forward and backward):
// the inverse scan order and the channel vectors the tile kernels move.
#pragma once
#include "dig_common.cuh"

namespace dig {

// Scan position of grid token (r, c): the inverse of the scan order.
__device__ __forceinline__ int grid_to_scan(int r, int c, int Hg, int Wg, int mode) {
  const int t = (mode & 2) ? c * Hg + r : r * Wg + c;
  return (mode & 1) ? Hg * Wg - 1 - t : t;
}

// CP consecutive channels as loaded (CP = 2 or 4): raw vector, unpack, store.
template <typename T, int CP>
struct Vec;
template <>
struct Vec<__nv_bfloat16, 2> {
  using type = uint32_t;
  __device__ __forceinline__ static void unpack(uint32_t u, float* o) {
    o[0] = __uint_as_float(u << 16);
    o[1] = __uint_as_float(u & 0xFFFF0000u);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* v) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v[0], v[1]);
  }
};
template <>
struct Vec<__nv_bfloat16, 4> {
  using type = uint2;
  __device__ __forceinline__ static void unpack(uint2 u, float* o) {
    o[0] = __uint_as_float(u.x << 16);
    o[1] = __uint_as_float(u.x & 0xFFFF0000u);
    o[2] = __uint_as_float(u.y << 16);
    o[3] = __uint_as_float(u.y & 0xFFFF0000u);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* v) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
  }
};
template <>
struct Vec<float, 2> {
  using type = float2;
  __device__ __forceinline__ static void unpack(float2 u, float* o) {
    o[0] = u.x;
    o[1] = u.y;
  }
  __device__ __forceinline__ static void store(float* p, const float* v) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  }
};
template <>
struct Vec<float, 4> {
  using type = float4;
  __device__ __forceinline__ static void unpack(float4 u, float* o) {
    o[0] = u.x;
    o[1] = u.y;
    o[2] = u.z;
    o[3] = u.w;
  }
  __device__ __forceinline__ static void store(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

}  // namespace dig
