// srem.cu -- SREM reorient + 3x3 depthwise conv (DiG slides, "SREM (Spatial
// Reorient & Enhancement Module) の導入"; paper section "DiG Block").
//
//   y[b, t, ch] = bias[ch] + sum_{di,dj in {-1,0,1}} w[ch, di+1, dj+1] * x[b, r+di, c+dj, ch]
//   with (r, c) the grid coordinates of pi(t) and zero padding outside the grid.
//
// The conv input is read in grid order and the result is written directly in
// scan order, so the reorient costs no extra pass.  HBM-bound: each thread owns
// a 16-byte channel vector of one output token and reads the nine neighbouring
// vectors (the 9x reuse is served by L1/L2; DRAM sees x about once).  A block
// covers consecutive scan positions, which are grid neighbours in every mode.
#include "dig_common.cuh"
#include "gla.h"

namespace dig {

template <typename TIN, typename TOUT, int VEC>
__global__ void __launch_bounds__(256) srem_dwconv_kernel(const TIN* __restrict__ x, const float* __restrict__ w,
                                                          const float* __restrict__ bias, TOUT* __restrict__ y,
                                                          int B, int Hg, int Wg, int C, int mode) {
  const int L = Hg * Wg;
  const int ngrp = C / VEC;
  const long long total = (long long)B * L * ngrp;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int grp = (int)(idx % ngrp);
    const long long bt = idx / ngrp;
    const int t = (int)(bt % L);
    const int b = (int)(bt / L);
    const int g = scan_to_grid(t, L, Hg, Wg, mode);
    const int r0 = g / Wg, c0 = g - r0 * Wg;
    const int ch0 = grp * VEC;
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = bias ? __ldg(bias + ch0 + i) : 0.f;
#pragma unroll
    for (int di = -1; di <= 1; ++di) {
      const int rr = r0 + di;
      if (rr < 0 || rr >= Hg) continue;
#pragma unroll
      for (int dj = -1; dj <= 1; ++dj) {
        const int cc = c0 + dj;
        if (cc < 0 || cc >= Wg) continue;
        float xv[VEC];
        const TIN* src = x + (((long long)b * Hg + rr) * Wg + cc) * C + ch0;
        if constexpr (VEC >= 4) {
          load_row<VEC>(src, xv);
        } else {
#pragma unroll
          for (int i = 0; i < VEC; ++i) xv[i] = static_cast<float>(src[i]);
        }
        const int tap = (di + 1) * 3 + (dj + 1);
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] = fmaf(__ldg(w + (ch0 + i) * 9 + tap), xv[i], acc[i]);
      }
    }
    TOUT* dst = y + ((long long)b * L + t) * C + ch0;
    if constexpr (VEC >= 4) {
      store_row<VEC>(dst, acc);
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) dst[i] = static_cast<TOUT>(acc[i]);
    }
  }
}

template <typename TIN, typename TOUT>
static cudaError_t launch_typed(const void* x, const float* w, const float* bias, void* y, int B, int Hg, int Wg,
                                int C, int mode, cudaStream_t s) {
  constexpr int VEC = 16 / sizeof(TIN);  // one 16-byte vector of input channels
  const long long L = (long long)Hg * Wg;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (C % VEC == 0) {
    const long long work = (long long)B * L * (C / VEC);
    const long long blocks = (work + 255) / 256;
    const int grid = (int)(blocks < (long long)sms * 16 ? blocks : (long long)sms * 16);
    srem_dwconv_kernel<TIN, TOUT, VEC><<<grid, 256, 0, s>>>(reinterpret_cast<const TIN*>(x), w, bias,
                                                             reinterpret_cast<TOUT*>(y), B, Hg, Wg, C, mode);
  } else {
    const long long work = (long long)B * L * C;
    const long long blocks = (work + 255) / 256;
    const int grid = (int)(blocks < (long long)sms * 16 ? blocks : (long long)sms * 16);
    srem_dwconv_kernel<TIN, TOUT, 1><<<grid, 256, 0, s>>>(reinterpret_cast<const TIN*>(x), w, bias,
                                                           reinterpret_cast<TOUT*>(y), B, Hg, Wg, C, mode);
  }
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
