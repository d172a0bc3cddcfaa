// srem_bwd.cu -- backward of the SREM reorient + 3x3 depthwise conv (DiG slides,
// "SREM (Spatial Reorient & Enhancement Module) の導入"; paper section "DiG Block").
//
// The forward is y[b, t] = bias + sum_{di,dj} w[di+1, dj+1] x[b, pi(t) + (di, dj)]
// (zero padding, y in scan order).  With dyg[b, g] = dy[b, pi^-1(g)] the scan-order
// gradient read at grid token g:
//   dx[b, g]        = sum_{di,dj} w[di+1, dj+1] dyg[b, g - (di, dj)]   (terms inside the grid)
//   dw[ch, di, dj]  = sum_{b,g} dyg[b, g] x[b, g + (di, dj)]
//   dbias[ch]       = sum_{b,g} dyg[b, g]
// One pass reads dy (scan order) and x (grid order) once from HBM and writes dx in
// grid order; the weight and bias gradients are reduced on chip.
#include "dig_common.cuh"
#include "bwd_ops.h"
#include "gla_common.cuh"
#include "srem.cuh"

namespace dig {

// 4- or 8-byte asynchronous global -> shared copy, zero-filled when !valid (no
// bytes are read then; src must still be a valid address).
template <int BYTES>
__device__ __forceinline__ void cp_async_zfill(uint32_t saddr, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(saddr), "l"(src), "n"(BYTES),
               "r"(valid ? BYTES : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Tile kernel (2 channels per thread).  A block is 8 warps over 32 channel pairs:
// lane l owns channel pair (slab * 32 + l), warp w owns TW adjacent grid columns,
// so a warp access is 32 consecutive channel pairs of one pixel (contiguous) and
// the block's warps cover 8 * TW adjacent columns.  A work item is R grid rows of
// those columns for one image; the blocks of a channel slab stride over the items
// (the grid is the number of resident blocks), so each thread keeps its 9 x 2
// weight-gradient and 2 bias-gradient partials in registers across items.
// Per item a thread copies its (R + 2) x (TW + 2) windows of dy (at the scan
// positions of the grid pixels: a base plus constant steps per grid row and
// column, as in the forward) and of x into its own shared-memory slots with
// cp.async, zero-filled outside the grid.  The copies of the next item are in
// flight while the current one is computed (two stages; each thread reads only
// the slots it filled, so no block barrier is needed).  The compute walks down
// the rows with 3-row register windows.  At the end the 8 warps' partials are
// summed in shared memory and each block adds them to dw / dbias with one atomic
// per value.
template <typename TIN, typename TOUT, int TW, int R, int MINB>
__global__ void __launch_bounds__(256, MINB)
    srem_dwconv_bwd_kernel(const TIN* __restrict__ x, const float* __restrict__ w, const TIN* __restrict__ dy,
                           TOUT* __restrict__ dx, float* __restrict__ dw, float* __restrict__ dbias, int B, int Hg,
                           int Wg, int C, int mode, int nslab, int per_slab, int ncs, int nrt) {
  constexpr int CP = 2, NV = 10 * CP;    // 9 taps + bias, per channel
  constexpr int NW = (R + 2) * (TW + 2);  // window pixels
  using VT = typename Vec<TIN, CP>::type;
  constexpr int VB = (int)sizeof(VT);
  // stage[s][warp][tensor: 0 dy, 1 x][window pixel][lane]
  extern __shared__ __align__(16) unsigned char conv_bwd_smem[];
  VT* stage = reinterpret_cast<VT*>(conv_bwd_smem);
  __shared__ float red[NV][32];
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < NV * 32; i += blockDim.x) (&red[0][0])[i] = 0.f;
  const int slab = blockIdx.x % nslab;
  const int nv = C / CP;
  const int chv = slab * 32 + lane;
  const bool ch_ok = chv < nv;
  const int ch = CP * (ch_ok ? chv : 0);
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
  float gw[9][CP], gb[CP];
#pragma unroll
  for (int e = 0; e < CP; ++e) {
    gb[e] = 0.f;
#pragma unroll
    for (int tap = 0; tap < 9; ++tap) gw[tap][e] = 0.f;
  }
  const int L = Hg * Wg;
  const int sgn = (mode & 1) ? -1 : 1;
  const ptrdiff_t rstep = (ptrdiff_t)sgn * ((mode & 2) ? 1 : Wg) * C;  // dy elements per grid row
  const ptrdiff_t cstep = (ptrdiff_t)sgn * ((mode & 2) ? Hg : 1) * C;  // dy elements per grid column
  const bool want_w = dw || dbias;  // x is read only then (it may be NULL otherwise)
  const int items = ncs * nrt * B;
  // shared-memory address of window pixel e of tensor tn in stage st (this thread's slot)
  const uint32_t slot0 = smem_u32(stage) + (uint32_t)((warp * 2 * NW) * 32 + lane) * VB;
  auto slot = [&](int st, int tn, int e) -> uint32_t {
    return slot0 + (uint32_t)(((st * 8 * 2 * NW) + tn * NW + e) * 32) * VB;
  };
  auto item_origin = [&](int it, int& b, int& r0, int& c0) {
    const int cs = it % ncs, rest = it / ncs;
    r0 = (rest % nrt) * R;
    b = rest / nrt;
    c0 = (cs * 8 + warp) * TW;
  };
  auto issue = [&](int it, int st) {
    int b, r0, c0;
    item_origin(it, b, r0, c0);
    if (c0 >= Wg || !ch_ok) return;
    const TIN* dyb = dy + ((size_t)b * L + grid_to_scan(r0, c0, Hg, Wg, mode)) * C + ch;
    const TIN* xb = want_w ? x + (((size_t)b * Hg + r0) * Wg + c0) * C + ch : nullptr;
#pragma unroll
    for (int i = 0; i < R + 2; ++i) {
      const int rr = r0 - 1 + i;
      const bool rok = rr >= 0 && rr < Hg;
#pragma unroll
      for (int j = 0; j < TW + 2; ++j) {
        const int cc = c0 - 1 + j;
        const bool ok = rok && cc >= 0 && cc < Wg;
        const int e = i * (TW + 2) + j;
        cp_async_zfill<VB>(slot(st, 0, e), ok ? dyb + (ptrdiff_t)(i - 1) * rstep + (ptrdiff_t)(j - 1) * cstep : dy,
                           ok);
        if (want_w)
          cp_async_zfill<VB>(slot(st, 1, e), ok ? xb + ((ptrdiff_t)(i - 1) * Wg + (j - 1)) * C : x, ok);
      }
    }
  };
  auto load_row = [&](int st, int tn, int i, float (*dst)[CP]) {
#pragma unroll
    for (int j = 0; j < TW + 2; ++j) {
      VT v;
      if constexpr (VB == 4) {
        uint32_t u;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(u) : "r"(slot(st, tn, i * (TW + 2) + j)));
        v = u;
      } else {
        float2 u;
        asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                     : "=f"(u.x), "=f"(u.y)
                     : "r"(slot(st, tn, i * (TW + 2) + j)));
        v = u;
      }
      Vec<TIN, CP>::unpack(v, dst[j]);
    }
  };
  int it = blockIdx.x / nslab, st = 0;
  if (it < items) issue(it, 0);
  cp_async_commit();
  for (; it < items; it += per_slab, st ^= 1) {
    if (it + per_slab < items) issue(it + per_slab, st ^ 1);
    cp_async_commit();
    cp_async_wait_group<1>();  // this thread's copies of item `it` have landed
    int b, r0, c0;
    item_origin(it, b, r0, c0);
    if (c0 >= Wg || !ch_ok) continue;
    TOUT* out = dx + (((size_t)b * Hg + r0) * Wg + c0) * C + ch;
    float d0[TW + 2][CP], d1[TW + 2][CP], d2[TW + 2][CP];
    float x0[TW + 2][CP], x1[TW + 2][CP], x2[TW + 2][CP];
    load_row(st, 0, 0, d0);
    load_row(st, 0, 1, d1);
    if (want_w) {
      load_row(st, 1, 0, x0);
      load_row(st, 1, 1, x1);
    }
#pragma unroll
    for (int i = 0; i < R; ++i, out += (size_t)Wg * C) {
      load_row(st, 0, i + 2, d2);
      if (want_w) load_row(st, 1, i + 2, x2);
      // output pixel (r0+i, c0+k) sits at d1[k+1]; its dx reads dyg at offsets
      // -(di, dj), i.e. window rows 2..0 and columns k+2..k against taps 0..2
#pragma unroll
      for (int k = 0; k < TW; ++k) {
        float acc[CP];
#pragma unroll
        for (int e = 0; e < CP; ++e) {
          acc[e] = 0.f;
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            acc[e] = fmaf(wr[t][e], d2[k + 2 - t][e], acc[e]);
            acc[e] = fmaf(wr[3 + t][e], d1[k + 2 - t][e], acc[e]);
            acc[e] = fmaf(wr[6 + t][e], d0[k + 2 - t][e], acc[e]);
          }
          if (want_w) {
#pragma unroll
            for (int t = 0; t < 3; ++t) {
              gw[t][e] = fmaf(d1[k + 1][e], x0[k + t][e], gw[t][e]);
              gw[3 + t][e] = fmaf(d1[k + 1][e], x1[k + t][e], gw[3 + t][e]);
              gw[6 + t][e] = fmaf(d1[k + 1][e], x2[k + t][e], gw[6 + t][e]);
            }
            gb[e] += d1[k + 1][e];
          }
        }
        if (r0 + i < Hg && c0 + k < Wg) Vec<TOUT, CP>::store(out + (size_t)k * C, acc);
      }
#pragma unroll
      for (int j = 0; j < TW + 2; ++j)
#pragma unroll
        for (int e = 0; e < CP; ++e) {
          d0[j][e] = d1[j][e];
          d1[j][e] = d2[j][e];
          x0[j][e] = x1[j][e];
          x1[j][e] = x2[j][e];
        }
    }
  }
  cp_async_wait_group<0>();
  if (!want_w) return;
  __syncthreads();  // red zeroed
  if (ch_ok) {
#pragma unroll
    for (int e = 0; e < CP; ++e) {
#pragma unroll
      for (int tap = 0; tap < 9; ++tap) atomicAdd(&red[tap * CP + e][lane], gw[tap][e]);
      atomicAdd(&red[9 * CP + e][lane], gb[e]);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NV * 32; i += blockDim.x) {
    const int v = i >> 5, l = i & 31;
    const int cv = slab * 32 + l;
    if (cv >= nv) continue;
    const int tap = v / CP, c = CP * cv + v % CP;
    if (tap < 9) {
      if (dw) atomicAdd(dw + (size_t)c * 9 + tap, red[v][l]);
    } else if (dbias) {
      atomicAdd(dbias + c, red[v][l]);
    }
  }
}

// Odd channel counts: dx one thread per (pixel, channel) ...
template <typename TIN, typename TOUT>
__global__ void __launch_bounds__(256) srem_dwconv_bwd_dx_scalar_kernel(const float* __restrict__ w,
                                                                        const TIN* __restrict__ dy,
                                                                        TOUT* __restrict__ dx, int B, int Hg, int Wg,
                                                                        int C, int mode) {
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const long long total = (long long)B * Hg * Wg * C;
  const long long L = (long long)Hg * Wg;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(idx % C);
    const long long pix = idx / C;
    const int c = (int)(pix % Wg);
    const long long br = pix / Wg;
    const int r = (int)(br % Hg), b = (int)(br / Hg);
    float acc = 0.f;
    for (int di = -1; di <= 1; ++di)
      for (int dj = -1; dj <= 1; ++dj) {
        const int rr = r - di, cc = c - dj;
        if (rr < 0 || rr >= Hg || cc < 0 || cc >= Wg) continue;
        acc = fmaf(__ldg(w + ch * 9 + (di + 1) * 3 + (dj + 1)),
                   static_cast<float>(dy[((long long)b * L + grid_to_scan(rr, cc, Hg, Wg, mode)) * C + ch]), acc);
      }
    dx[idx] = static_cast<TOUT>(acc);
  }
}

// ... and one block per (channel, tap or bias) summing over all pixels (no atomics).
template <typename TIN>
__global__ void __launch_bounds__(256) srem_dwconv_bwd_dw_scalar_kernel(const TIN* __restrict__ x,
                                                                        const TIN* __restrict__ dy,
                                                                        float* __restrict__ dw,
                                                                        float* __restrict__ dbias, int B, int Hg,
                                                                        int Wg, int C, int mode) {
  __shared__ float part[8];
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const int ch = blockIdx.x / 10, tap = blockIdx.x % 10;
  if ((tap < 9 && !dw) || (tap == 9 && !dbias)) return;
  const int di = tap / 3 - 1, dj = tap % 3 - 1;
  const long long L = (long long)Hg * Wg;
  float acc = 0.f;
  for (long long p = threadIdx.x; p < (long long)B * L; p += blockDim.x) {
    const long long b = p / L;
    const int g = (int)(p % L), r = g / Wg, c = g % Wg;
    const float d = static_cast<float>(dy[(b * L + grid_to_scan(r, c, Hg, Wg, mode)) * C + ch]);
    if (tap == 9) {
      acc += d;
      continue;
    }
    const int xr = r + di, xc = c + dj;
    if (xr < 0 || xr >= Hg || xc < 0 || xc >= Wg) continue;
    acc = fmaf(d, static_cast<float>(x[((b * Hg + xr) * Wg + xc) * C + ch]), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < 8; ++i) s += part[i];
    if (tap < 9) dw[(size_t)ch * 9 + tap] = s;
    else dbias[ch] = s;
  }
}

// Tile shape of the backward: columns and rows per thread and resident blocks per
// SM.  The windows live in shared memory: 2 stages x 8 warps x 2 tensors x
// (R+2)(TW+2) pixels x 32 lanes x 4 bytes (bf16 channel pairs) = 96 KB per block
// for 2 x 4 tiles, two blocks per SM (the largest tile that compiles without
// register spills at that occupancy); fp32 pairs take twice the bytes per pixel,
// so fp32 inputs use 2 x 2 tiles (128 KB, one block per SM).
template <typename TIN>
struct ConvBwdTile {
  static constexpr int kCols = 2, kRows = sizeof(TIN) == 2 ? 4 : 2, kMinBlocks = sizeof(TIN) == 2 ? 2 : 1;
  static constexpr size_t kSmem = 2ull * 8 * 2 * (kRows + 2) * (kCols + 2) * 32 * 2 * sizeof(TIN);
};

template <typename TIN, typename TOUT>
static cudaError_t launch_bwd_typed(const void* x, const float* w, const void* dy, void* dx, float* dw, float* dbias,
                                    int B, int Hg, int Wg, int C, int mode, cudaStream_t s) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const TIN* xt = reinterpret_cast<const TIN*>(x);
  const TIN* dyt = reinterpret_cast<const TIN*>(dy);
  if (C % 2 != 0) {
    const long long total = (long long)B * Hg * Wg * C;
    const long long blocks = (total + 255) / 256;
    const int grid = (int)(blocks < (long long)sms * 32 ? blocks : (long long)sms * 32);
    cudaError_t e = launch_pdl(srem_dwconv_bwd_dx_scalar_kernel<TIN, TOUT>, dim3(grid), dim3(256), 0, s, w, dyt,
                               reinterpret_cast<TOUT*>(dx), B, Hg, Wg, C, mode);
    if (e != cudaSuccess || (!dw && !dbias)) return e;
    if ((long long)C * 10 > 2147483647LL) return cudaErrorInvalidValue;
    return launch_pdl(srem_dwconv_bwd_dw_scalar_kernel<TIN>, dim3(C * 10), dim3(256), 0, s, xt, dyt, dw, dbias, B,
                      Hg, Wg, C, mode);
  }
  using Tile = ConvBwdTile<TIN>;
  constexpr int TW = Tile::kCols, R = Tile::kRows, MINB = Tile::kMinBlocks;
  auto kern = srem_dwconv_bwd_kernel<TIN, TOUT, TW, R, MINB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Tile::kSmem);
  if (e != cudaSuccess) return e;
  if (dw) {
    e = cudaMemsetAsync(dw, 0, (size_t)C * 9 * sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  if (dbias) {
    e = cudaMemsetAsync(dbias, 0, (size_t)C * sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, Tile::kSmem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const long long nslab = (C / 2 + 31) / 32;
  const long long ncs = ((Wg + TW - 1) / TW + 7) / 8, nrt = (Hg + R - 1) / R;
  const long long items = ncs * nrt * B;
  if (items > 2147483647LL) return cudaErrorInvalidValue;
  // blocks per channel slab: as many as fit in one wave of resident blocks
  long long per_slab = (long long)sms * per_sm / nslab;
  if (per_slab < 1) per_slab = 1;
  if (per_slab > items) per_slab = items;
  if (nslab * per_slab > 2147483647LL) return cudaErrorInvalidValue;
  return launch_pdl(kern, dim3((unsigned)(nslab * per_slab)), dim3(256), Tile::kSmem, s, xt, w, dyt,
                    reinterpret_cast<TOUT*>(dx), dw, dbias, B, Hg, Wg, C, mode, (int)nslab, (int)per_slab, (int)ncs,
                    (int)nrt);
}

cudaError_t launch_srem_bwd(const void* x, const float* w, const void* dy, void* dx, float* dw, float* dbias, int B,
                            int Hg, int Wg, int C, int mode, int tin, int tout, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (tin == DIG_BF16) {
    if (tout == DIG_BF16) return launch_bwd_typed<bf, bf>(x, w, dy, dx, dw, dbias, B, Hg, Wg, C, mode, s);
    return launch_bwd_typed<bf, float>(x, w, dy, dx, dw, dbias, B, Hg, Wg, C, mode, s);
  }
  if (tout == DIG_BF16) return launch_bwd_typed<float, bf>(x, w, dy, dx, dw, dbias, B, Hg, Wg, C, mode, s);
  return launch_bwd_typed<float, float>(x, w, dy, dx, dw, dbias, B, Hg, Wg, C, mode, s);
}

}  // namespace dig
