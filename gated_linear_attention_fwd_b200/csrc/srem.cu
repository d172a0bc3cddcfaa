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

namespace dig {

// Scan position of grid token (r, c): the inverse of the scan order.
__device__ __forceinline__ int grid_to_scan(int r, int c, int Hg, int Wg, int mode) {
  const int t = (mode & 2) ? c * Hg + r : r * Wg + c;
  return (mode & 1) ? Hg * Wg - 1 - t : t;
}

// Row-streaming kernel.  A thread owns 2 consecutive channels of one grid
// column and kRows consecutive output rows.  It issues the loads of all
// kRows + 2 input rows x 3 columns it needs at once (consecutive lanes read
// consecutive channel pairs of one pixel, so every warp load is contiguous),
// then walks down the rows with a 3-row window unpacked once per row and the
// 9 x 2 weights in registers (one contiguous 72-byte run of w per thread).
// Consecutive grid rows of one column are a fixed step apart in every scan
// order, so the output pointer advances by a constant.
constexpr int kConvRows = 8;

template <typename T>
struct Pair;  // two consecutive channels as loaded
template <>
struct Pair<__nv_bfloat16> {
  using type = uint32_t;
  __device__ __forceinline__ static void unpack(uint32_t u, float* o) {
    o[0] = __uint_as_float(u << 16);
    o[1] = __uint_as_float(u & 0xFFFF0000u);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
  }
};
template <>
struct Pair<float> {
  using type = float2;
  __device__ __forceinline__ static void unpack(float2 u, float* o) {
    o[0] = u.x;
    o[1] = u.y;
  }
  __device__ __forceinline__ static void store(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
  }
};

template <typename TIN, typename TOUT>
__global__ void __launch_bounds__(256, 3) srem_dwconv_kernel(const TIN* __restrict__ x, const float* __restrict__ w,
                                                          const float* __restrict__ bias, TOUT* __restrict__ y,
                                                          int B, int Hg, int Wg, int C, int mode) {
  constexpr int R = kConvRows;
  using PT = typename Pair<TIN>::type;
  const int np = C / 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int c = idx / np, ch = 2 * (idx - c * np);
  if (c >= Wg) return;
  const int b = blockIdx.z, r0 = blockIdx.y * R;
  const size_t pix = (size_t)C / 2;  // one pixel in units of PT
  // input rows r0-1 .. r0+R, columns c-1 .. c+1 (zero outside the grid)
  PT win[R + 2][3];
  {
    const bool cl = c > 0, cr = c + 1 < Wg;
    const PT* row = reinterpret_cast<const PT*>(x + (((size_t)b * Hg + r0 - 1) * Wg + c) * C + ch);
#pragma unroll
    for (int i = 0; i < R + 2; ++i, row += (size_t)Wg * pix) {
      const int rr = r0 - 1 + i;
      const bool rok = rr >= 0 && rr < Hg;
      win[i][0] = (rok && cl) ? __ldg(row - pix) : PT{};
      win[i][1] = rok ? __ldg(row) : PT{};
      win[i][2] = (rok && cr) ? __ldg(row + pix) : PT{};
    }
  }
  // the 9 taps of the two channels: 18 consecutive floats, 8-byte aligned
  float wr[9][2];
  {
    const float2* wp = reinterpret_cast<const float2*>(w + (size_t)ch * 9);
    float f[18];
#pragma unroll
    for (int i = 0; i < 9; ++i) {
      const float2 v = __ldg(wp + i);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
#pragma unroll
    for (int tap = 0; tap < 9; ++tap) {
      wr[tap][0] = f[tap];
      wr[tap][1] = f[9 + tap];
    }
  }
  const float2 bv = bias ? __ldg(reinterpret_cast<const float2*>(bias + ch)) : make_float2(0.f, 0.f);
  // scan position of (r0, c) and its step per grid row
  const int L = Hg * Wg;
  const int t0 = grid_to_scan(r0 < Hg ? r0 : 0, c, Hg, Wg, mode);
  const int step = (mode & 2) ? 1 : Wg;
  const int sstep = (mode & 1) ? -step : step;
  TOUT* out = y + ((size_t)b * L + t0) * C + ch;
  const ptrdiff_t ostep = (ptrdiff_t)sstep * C;
  float u0[3][2], u1[3][2], u2[3][2];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    Pair<TIN>::unpack(win[0][j], u0[j]);
    Pair<TIN>::unpack(win[1][j], u1[j]);
  }
#pragma unroll
  for (int i = 0; i < R; ++i, out += ostep) {
#pragma unroll
    for (int j = 0; j < 3; ++j) Pair<TIN>::unpack(win[i + 2][j], u2[j]);
    if (r0 + i < Hg) {
      float a0 = bv.x, a1 = bv.y;
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        a0 = fmaf(wr[j][0], u0[j][0], a0);
        a1 = fmaf(wr[j][1], u0[j][1], a1);
        a0 = fmaf(wr[3 + j][0], u1[j][0], a0);
        a1 = fmaf(wr[3 + j][1], u1[j][1], a1);
        a0 = fmaf(wr[6 + j][0], u2[j][0], a0);
        a1 = fmaf(wr[6 + j][1], u2[j][1], a1);
      }
      Pair<TOUT>::store(out, a0, a1);
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      u0[j][0] = u1[j][0]; u0[j][1] = u1[j][1];
      u1[j][0] = u2[j][0]; u1[j][1] = u2[j][1];
    }
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
  if (C % 2 != 0) {  // channels that do not pair up
    const long long total = (long long)B * Hg * Wg * C;
    const long long blocks = (total + 255) / 256;
    const int grid = (int)(blocks < 148LL * 32 ? blocks : 148LL * 32);
    srem_dwconv_scalar_kernel<TIN, TOUT><<<grid, 256, 0, s>>>(reinterpret_cast<const TIN*>(x), w, bias,
                                                               reinterpret_cast<TOUT*>(y), B, Hg, Wg, C, mode);
    return cudaGetLastError();
  }
  constexpr int R = kConvRows;
  const long long gx = ((long long)Wg * (C / 2) + 255) / 256;
  const long long gy = (Hg + R - 1) / R;
  if (gx > 2147483647LL || gy > 65535 || B > 65535) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)gx, (unsigned)gy, (unsigned)B);
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
