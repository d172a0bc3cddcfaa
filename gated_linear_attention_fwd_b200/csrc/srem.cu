// srem.cu -- SREM reorient + 3x3 depthwise conv (DiG slides, "SREM (Spatial
// Reorient & Enhancement Module) の導入"; paper section "DiG Block").
//
//   y[b, t, ch] = bias[ch] + sum_{di,dj in {-1,0,1}} w[ch, di+1, dj+1] * x[b, r+di, c+dj, ch]
//   with (r, c) the grid coordinates of pi(t) and zero padding outside the grid.
//
// The conv input is read in grid order and the result is written directly in
// scan order, so the reorient costs no extra pass.  HBM-bound; see the kernel
// comment for the traversal.
#include "dig_common.cuh"
#include "gla.h"

namespace dig {

// Raw 16-byte vector of VEC input channels, unpacked to fp32 on use.
template <typename T>
__device__ __forceinline__ void unpack_vec(const uint4& u, float* o);
template <>
__device__ __forceinline__ void unpack_vec<__nv_bfloat16>(const uint4& u, float* o) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void unpack_vec<float>(const uint4& u, float* o) {
  o[0] = __uint_as_float(u.x);
  o[1] = __uint_as_float(u.y);
  o[2] = __uint_as_float(u.z);
  o[3] = __uint_as_float(u.w);
}

// Scan position of grid token (r, c): the inverse of the scan order.
__device__ __forceinline__ int grid_to_scan(int r, int c, int Hg, int Wg, int mode) {
  const int t = (mode & 2) ? c * Hg + r : r * Wg + c;
  return (mode & 1) ? Hg * Wg - 1 - t : t;
}

// Shared-memory tile: a block produces an 8 x 32 pixel tile of one image for
// one 128-byte slice of channels.  It first loads the tile plus its one-pixel
// halo (10 x 34 pixels x 128 bytes) with 16-byte loads issued together, then
// each thread computes 8 outputs of one 16-byte channel vector from shared
// memory (its 9 x VEC weights stay in registers) and stores them at their scan
// positions.  HBM reads are the tile plus halo (~1.33x the output tile).
constexpr int kTR = 8, kTC = 32, kSliceBytes = 128;

template <typename TIN, typename TOUT>
__global__ void __launch_bounds__(256) srem_dwconv_kernel(const TIN* __restrict__ x, const float* __restrict__ w,
                                                          const float* __restrict__ bias, TOUT* __restrict__ y,
                                                          int B, int Hg, int Wg, int C, int mode) {
  constexpr int VEC = 16 / sizeof(TIN);
  constexpr int CS = kSliceBytes / sizeof(TIN);  // channels per slice
  constexpr int NV = kSliceBytes / 16;            // 16-byte vectors per pixel-slice (8)
  constexpr int TW = kTC + 2, TH = kTR + 2;
  __shared__ uint4 tile[TH * TW * NV];
  const int nslice = (C + CS - 1) / CS;
  const int b = blockIdx.z / nslice, slice = blockIdx.z - b * nslice;
  const int ch_base = slice * CS;
  const int r0 = blockIdx.y * kTR, c0 = blockIdx.x * kTC;
  const TIN* img = x + (size_t)b * Hg * Wg * C;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < TH * TW * NV; i += blockDim.x) {
    const int v = i % NV, pix = i / NV;
    const int rr = r0 - 1 + pix / TW, cc = c0 - 1 + pix % TW, ch = ch_base + v * VEC;
    uint4 u = zero;
    if (rr >= 0 && rr < Hg && cc >= 0 && cc < Wg && ch < C)
      u = __ldg(reinterpret_cast<const uint4*>(img + ((size_t)rr * Wg + cc) * C + ch));
    tile[i] = u;
  }
  __syncthreads();
  const int v = threadIdx.x % NV;
  const int ch0 = ch_base + v * VEC;
  if (ch0 >= C) return;
  float wr[9][VEC], bv[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    bv[i] = bias ? __ldg(bias + ch0 + i) : 0.f;
#pragma unroll
    for (int tap = 0; tap < 9; ++tap) wr[tap][i] = __ldg(w + (ch0 + i) * 9 + tap);
  }
  for (int pix = threadIdx.x / NV; pix < kTR * kTC; pix += blockDim.x / NV) {
    const int tr = pix / kTC, tc = pix % kTC;
    const int r = r0 + tr, c = c0 + tc;
    if (r >= Hg || c >= Wg) continue;
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = bv[i];
#pragma unroll
    for (int di = 0; di < 3; ++di) {
#pragma unroll
      for (int dj = 0; dj < 3; ++dj) {
        float xv[VEC];
        unpack_vec<TIN>(tile[((tr + di) * TW + (tc + dj)) * NV + v], xv);
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] = fmaf(wr[di * 3 + dj][i], xv[i], acc[i]);
      }
    }
    store_row<VEC>(y + ((size_t)b * Hg * Wg + grid_to_scan(r, c, Hg, Wg, mode)) * C + ch0, acc);
  }
}

// Channels that do not fill 16-byte vectors: one thread per (token, channel).
template <typename TIN, typename TOUT>
__global__ void __launch_bounds__(256) srem_dwconv_scalar_kernel(const TIN* __restrict__ x,
                                                                 const float* __restrict__ w,
                                                                 const float* __restrict__ bias, TOUT* __restrict__ y,
                                                                 int B, int Hg, int Wg, int C, int mode) {
  const long long total = (long long)B * Hg * Wg * C;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(idx % C);
    const long long pix = idx / C;
    const int c = (int)(pix % Wg);
    const long long br = pix / Wg;
    const int r = (int)(br % Hg), b = (int)(br / Hg);
    float acc = bias ? __ldg(bias + ch) : 0.f;
    for (int di = -1; di <= 1; ++di)
      for (int dj = -1; dj <= 1; ++dj) {
        const int rr = r + di, cc = c + dj;
        if (rr < 0 || rr >= Hg || cc < 0 || cc >= Wg) continue;
        acc = fmaf(__ldg(w + ch * 9 + (di + 1) * 3 + (dj + 1)),
                   static_cast<float>(x[(((long long)b * Hg + rr) * Wg + cc) * C + ch]), acc);
      }
    y[((long long)b * Hg * Wg + grid_to_scan(r, c, Hg, Wg, mode)) * C + ch] = static_cast<TOUT>(acc);
  }
}

template <typename TIN, typename TOUT>
static cudaError_t launch_typed(const void* x, const float* w, const float* bias, void* y, int B, int Hg, int Wg,
                                int C, int mode, cudaStream_t s) {
  constexpr int VEC = 16 / sizeof(TIN);  // one 16-byte vector of input channels
  if (C % VEC != 0) {
    const long long total = (long long)B * Hg * Wg * C;
    const long long blocks = (total + 255) / 256;
    const int grid = (int)(blocks < 148LL * 32 ? blocks : 148LL * 32);
    srem_dwconv_scalar_kernel<TIN, TOUT><<<grid, 256, 0, s>>>(reinterpret_cast<const TIN*>(x), w, bias,
                                                               reinterpret_cast<TOUT*>(y), B, Hg, Wg, C, mode);
    return cudaGetLastError();
  }
  const long long nz = (long long)B * ((C + kSliceBytes / (int)sizeof(TIN) - 1) / (kSliceBytes / (int)sizeof(TIN)));
  if (nz > 65535 || (Hg + kTR - 1) / kTR > 65535) return cudaErrorInvalidValue;
  const dim3 grid((Wg + kTC - 1) / kTC, (Hg + kTR - 1) / kTR, (unsigned)nz);
  srem_dwconv_kernel<TIN, TOUT><<<grid, 256, 0, s>>>(reinterpret_cast<const TIN*>(x), w, bias,
                                                      reinterpret_cast<TOUT*>(y), B, Hg, Wg, C, mode);
  return cudaGetLastError();
}

cudaError_t launch_srem(const void* x, const float* w, const float* bias, void* y, int B, int Hg, int Wg, int C,
                        int mode, int tin, int tout, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (tin == DIG_BF16) {
    if (tout == DIG_BF16) return launch_typed<bf, bf>(x, w, bias, y, B, Hg, Wg, C, mode, s);
    return launch_typed<bf, float>(x, w, bias, y, B, Hg, Wg, C, mode, s);
  }
  if (tout == DIG_BF16) return launch_typed<float, bf>(x, w, bias, y, B, Hg, Wg, C, mode, s);
  return launch_typed<float, float>(x, w, bias, y, B, Hg, Wg, C, mode, s);
}

}  // namespace dig
