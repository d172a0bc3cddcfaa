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
#include "gla_common.cuh"
#include "srem.cuh"

namespace dig {

// Tile kernel.  A thread owns 2 consecutive channels of TW adjacent grid
// columns and R consecutive output rows.  It issues the loads of all R + 2
// input rows x TW + 2 columns it needs at once (consecutive lanes read
// consecutive channel pairs of one pixel, so every warp load is contiguous;
// adjacent columns share their neighbours' loads), then walks down the rows
// with a 3-row window unpacked once per row and the 9 x 2 weights in registers
// (one contiguous 72-byte run of w per thread).  Neighbouring grid pixels are a
// fixed step apart in scan order along a row and along a column in every scan
// order, so output addresses are a base plus constant steps.
template <typename TIN, typename TOUT, int CP, int TW, int R, int MINB>
__global__ void __launch_bounds__(256, MINB) srem_dwconv_kernel(const TIN* __restrict__ x, const float* __restrict__ w,
                                                             const float* __restrict__ bias, TOUT* __restrict__ y,
                                                             int B, int Hg, int Wg, int C, int mode) {
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  using VT = typename Vec<TIN, CP>::type;
  const int nv = C / CP;  // channel vectors per pixel
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int cg = idx / nv, ch = CP * (idx - cg * nv);
  const int c0 = cg * TW;
  if (c0 >= Wg) return;
  const int b = blockIdx.z, r0 = blockIdx.y * R;
  const size_t pix = (size_t)nv;  // one pixel in units of VT
  // input rows r0-1 .. r0+R, columns c0-1 .. c0+TW (zero outside the grid)
  VT win[R + 2][TW + 2];
  {
    const VT* row = reinterpret_cast<const VT*>(x + (((size_t)b * Hg + r0 - 1) * Wg + c0) * C + ch);
#pragma unroll
    for (int i = 0; i < R + 2; ++i, row += (size_t)Wg * pix) {
      const int rr = r0 - 1 + i;
      const bool rok = rr >= 0 && rr < Hg;
#pragma unroll
      for (int j = 0; j < TW + 2; ++j) {
        const int cc = c0 - 1 + j;
        win[i][j] = (rok && cc >= 0 && cc < Wg) ? __ldg(row + (ptrdiff_t)(j - 1) * (ptrdiff_t)pix) : VT{};
      }
    }
  }
  // the 9 taps of the CP channels: 9 CP consecutive floats, 8-byte aligned
  float wr[9][CP];
  {
    const float2* wp = reinterpret_cast<const float2*>(w + (size_t)ch * 9);
    float f[9 * CP];
#pragma unroll
    for (int i = 0; i < 9 * CP / 2; ++i) {
      const float2 v = __ldg(wp + i);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
#pragma unroll
    for (int tap = 0; tap < 9; ++tap)
#pragma unroll
      for (int e = 0; e < CP; ++e) wr[tap][e] = f[9 * e + tap];
  }
  float bv[CP];
#pragma unroll
  for (int e = 0; e < CP; ++e) bv[e] = bias ? __ldg(bias + ch + e) : 0.f;
  // scan position of (r0, c0) and its steps per grid row and per grid column
  const int L = Hg * Wg;
  const int t0 = grid_to_scan(r0 < Hg ? r0 : 0, c0, Hg, Wg, mode);
  const int sgn = (mode & 1) ? -1 : 1;
  const ptrdiff_t rstep = (ptrdiff_t)sgn * ((mode & 2) ? 1 : Wg) * C;
  const ptrdiff_t cstep = (ptrdiff_t)sgn * ((mode & 2) ? Hg : 1) * C;
  TOUT* out = y + ((size_t)b * L + t0) * C + ch;
  float u0[TW + 2][CP], u1[TW + 2][CP], u2[TW + 2][CP];
#pragma unroll
  for (int j = 0; j < TW + 2; ++j) {
    Vec<TIN, CP>::unpack(win[0][j], u0[j]);
    Vec<TIN, CP>::unpack(win[1][j], u1[j]);
  }
#pragma unroll
  for (int i = 0; i < R; ++i, out += rstep) {
#pragma unroll
    for (int j = 0; j < TW + 2; ++j) Vec<TIN, CP>::unpack(win[i + 2][j], u2[j]);
    if (r0 + i < Hg) {
#pragma unroll
      for (int k = 0; k < TW; ++k) {
        if (c0 + k < Wg) {
          float acc[CP];
#pragma unroll
          for (int e = 0; e < CP; ++e) {
            acc[e] = bv[e];
#pragma unroll
            for (int j = 0; j < 3; ++j) {
              acc[e] = fmaf(wr[j][e], u0[k + j][e], acc[e]);
              acc[e] = fmaf(wr[3 + j][e], u1[k + j][e], acc[e]);
              acc[e] = fmaf(wr[6 + j][e], u2[k + j][e], acc[e]);
            }
          }
          Vec<TOUT, CP>::store(out + k * cstep, acc);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < TW + 2; ++j)
#pragma unroll
      for (int e = 0; e < CP; ++e) {
        u0[j][e] = u1[j][e];
        u1[j][e] = u2[j][e];
      }
  }
}

// Channels that do not fill 16-byte vectors: one thread per (token, channel).
template <typename TIN, typename TOUT>
__global__ void __launch_bounds__(256) srem_dwconv_scalar_kernel(const TIN* __restrict__ x,
                                                                 const float* __restrict__ w,
                                                                 const float* __restrict__ bias, TOUT* __restrict__ y,
                                                                 int B, int Hg, int Wg, int C, int mode) {
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
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

// Tile shape of the conv kernel: channels, columns and rows per thread, and
// resident blocks per SM (2 channels x 4 columns x 8 rows measured fastest of
// the shapes with 2 or 4 channels, 1 to 4 columns and 4 to 16 rows on B200).
constexpr int kConvCh = 2, kConvCols = 4, kConvRows = 8, kConvMinBlocks = 1;

template <typename TIN, typename TOUT>
static cudaError_t launch_typed(const void* x, const float* w, const float* bias, void* y, int B, int Hg, int Wg,
                                int C, int mode, cudaStream_t s) {
  if (C % kConvCh != 0) {  // channels that do not fill the vectors
    const long long total = (long long)B * Hg * Wg * C;
    const long long blocks = (total + 255) / 256;
    const int grid = (int)(blocks < 148LL * 32 ? blocks : 148LL * 32);
    return launch_pdl(srem_dwconv_scalar_kernel<TIN, TOUT>, dim3(grid), dim3(256), 0, s,
                      reinterpret_cast<const TIN*>(x), w, bias, reinterpret_cast<TOUT*>(y), B, Hg, Wg, C, mode);
  }
  constexpr int CP = kConvCh, TW = kConvCols, R = kConvRows;
  const long long gx = ((long long)((Wg + TW - 1) / TW) * (C / CP) + 255) / 256;
  const long long gy = (Hg + R - 1) / R;
  if (gx > 2147483647LL || gy > 65535 || B > 65535) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)gx, (unsigned)gy, (unsigned)B);
  return launch_pdl(srem_dwconv_kernel<TIN, TOUT, CP, TW, R, kConvMinBlocks>, grid, dim3(256), 0, s,
                    reinterpret_cast<const TIN*>(x), w, bias, reinterpret_cast<TOUT*>(y), B, Hg, Wg, C, mode);
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
