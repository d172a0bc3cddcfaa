// gate_proj_bwd_tc.cu -- backward of the gate logits' low-rank projection on the
// tensor cores (DiG slides, "Gated Linear Attention Transformer (GLA) の導入",
// eq. (5): the key gate is sigmoid of a low-rank projection D -> R -> d_k of the
// block input; u = x W1, z = u W2 + b).  With dz = d log alpha * inv_tau *
// sigmoid(-z) (log alpha = inv_tau * logsigmoid(z)):
//
//   du = dz W2^T [rows, R],  dx = du W1^T [rows, D],
//   dW1 = x^T du [D, R],     dW2 = u^T dz [R, d_k],  db = sum of dz over the rows.
//
// dx and dW1 are 2 D R multiply-adds per token each against 4 D bytes of x and
// dx: products with an inner or outer dimension of R = 16, on the tensor cores.
// Per tile of 128 token rows:
//   * the x tile arrives by TMA as D / 64 boxes of 64 channels (bf16, 128-byte
//     swizzle);
//   * all threads form du on the CUDA cores from dz and W2 (fp32) and write it as
//     two bf16 terms (hi + lo) twice: token-major (A of dx, K = R) and
//     rank-major (B of dW1, K = tokens, the hi and lo terms as 32 rows);
//   * one thread issues dW1 += x^T [du_hi | du_lo] (A = the x boxes read MN-major,
//     M = 128 channels from two boxes, N = 32; the accumulators stay in TMEM for
//     the CTA's whole run) and dx = du W1^T (M = 128 tokens, N <= 256 per
//     product, the four hi/lo term pairs, so dx keeps fp32-level accuracy);
//   * the x buffer is refilled with the next tile, and the next tile's d log alpha,
//     z and u rows are requested, while all warps read dx from TMEM and store it
//     (through shared memory, whole 128-byte lines per store instruction);
//   * dW2 and db are summed per warp over its 16 tokens of every tile.
// At the end the CTA adds its dW1 (hi + lo halves), dW2 and db partials into the
// outputs with 16-byte atomics.  bf16 x, R <= 16 and d_k <= 32 (both multiples of
// 4), D a multiple of 128 up to 384 take this kernel (DiG-S's 384 -> 16 -> 32);
// other shapes run the CUDA-core kernel of gate_proj.cu.
#include "gate_proj.h"
#include "tma.cuh"
#include "tma_tiles.cuh"
#include "tmap.h"

namespace dig {

int num_sms();  // gla_fwd.cu

namespace {

constexpr int kBM = 128, kKB = 64;  // tokens per tile, channels per x box
constexpr uint32_t kXB = kBM * kKB * 2;  // bytes of one x box (16 KB)
constexpr int kMaxD = 384, kMaxDK = 32;
constexpr uint32_t kTmDW1 = 384;  // TMEM column of the dW1 accumulators (32 per 128-channel block)

struct GbSmem {
  uint64_t xfull, mma_done;
  uint32_t tmem;
  int abort;
};

// Dynamic shared memory (offsets from a 1024-byte aligned base):
//   x      D / 64 boxes of [128 tokens][64 channels] bf16, 128-byte swizzle
//   w1     W1^T terms: [N = D][K = 16] bf16, no swizzle, K-major (core matrices
//          8 rows x 16 B; LBO 128, SBO 256), hi then lo
//   dua    du terms [M = 128 tokens][K = 16] bf16 (same layout), hi then lo
//   dub    du^T [N = 32: r hi, then r lo][K = 128 tokens] bf16, no swizzle (LBO 128, SBO 2048)
//   dz     [128][d_k + 1] fp32;  us [128][20] fp32 (16-byte rows);  w2 W2^T [d_k][16] fp32
//   stage  dx staging, 4 KB per warp (32 rows x 128 bytes)
struct GbLayout {
  uint32_t x, w1, dua, dub, dz, us, w2, stage, total;
  __host__ __device__ GbLayout(int D, int dk) {
    x = 0;
    w1 = (uint32_t)(D / kKB) * kXB;
    dua = w1 + 2u * (uint32_t)(D / 8) * 256u;
    dub = dua + 2u * 4096u;
    dz = dub + 8192u;
    us = dz + (uint32_t)kBM * (dk + 1) * 4u;
    w2 = us + (uint32_t)kBM * 20u * 4u;
    stage = (w2 + 16u * (uint32_t)dk * 4u + 127u) & ~127u;
    total = stage + 8u * 4096u;
  }
};

// Byte offset of element (row, k) in a no-swizzle K-major bf16 operand.
__device__ __forceinline__ uint32_t kmaj(int row, int k, uint32_t lbo, uint32_t sbo) {
  return (uint32_t)(row >> 3) * sbo + (uint32_t)(k >> 3) * lbo + (uint32_t)(row & 7) * 16u + (uint32_t)(k & 7) * 2u;
}

__device__ __forceinline__ float sigmoid_of_neg(float z) { return __fdividef(1.f, 1.f + ex2(z * kLog2e)); }

__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

__device__ __forceinline__ void store32(float* p, const float* v) {
#pragma unroll
  for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}
__device__ __forceinline__ void store32(__nv_bfloat16* p, const float* v) {
#pragma unroll
  for (int i = 0; i < 32; i += 8)
    *reinterpret_cast<uint4*>(p + i) = make_uint4(pack_bf16x2(v[i], v[i + 1]), pack_bf16x2(v[i + 2], v[i + 3]),
                                                  pack_bf16x2(v[i + 4], v[i + 5]), pack_bf16x2(v[i + 6], v[i + 7]));
}

template <typename TOUT>
__global__ void __launch_bounds__(256, 1) gate_proj_bwd_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                  const float* __restrict__ W1,
                                                                  const float* __restrict__ W2,
                                                                  const float* __restrict__ u,
                                                                  const float* __restrict__ z,
                                                                  const float* __restrict__ dla, float inv_tau,
                                                                  TOUT* __restrict__ dx, float* __restrict__ dW1,
                                                                  float* __restrict__ dW2, float* __restrict__ db,
                                                                  long long rows, int D, int R, int dk,
                                                                  uint32_t* status) {
  constexpr int NLD = kMaxDK / 8;        // 16-byte loads of d log alpha (and of z) per thread and tile
  extern __shared__ uint8_t smem_raw[];
  __shared__ GbSmem sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sb - smem_u32(smem_raw));
  const GbLayout lay(D, dk);
  const int nkb = D / kKB, nmb = D / 128;
  const int nh = D <= 256 ? 1 : 2, NH = D / nh;  // dx products per tile and their width
  const long long ntiles = (rows + kBM - 1) / kBM;
  const int mytiles = blockIdx.x < ntiles ? (int)((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  float* DZ = reinterpret_cast<float*>(sgen + lay.dz);
  float* US = reinterpret_cast<float*>(sgen + lay.us);
  float* W2S = reinterpret_cast<float*>(sgen + lay.w2);
  if (warp == 0) {
    tmem_alloc(&sh.tmem, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sh.xfull, 1);
    mbar_init(&sh.mma_done, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();  // the barriers are initialised before any thread waits on them
  tc_fence_after();
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  auto tile_row = [&](int i) { return (long long)(blockIdx.x + (long long)i * gridDim.x) * kBM; };
  auto load_x = [&](int i) {  // thread 0
    mbar_arrive_expect_tx(&sh.xfull, (uint32_t)nkb * kXB);
    for (int kb = 0; kb < nkb; ++kb) tma_load_2d(sb + lay.x + kb * kXB, xmap, kb * kKB, (int)tile_row(i), &sh.xfull);
  };
  // thread 0's record of the asynchronous work in flight, drained before exit
  int x_pending = 0, mma_pending = 0;  // an x tile requested / products committed, not yet seen complete
  uint32_t x_par = 0, mma_par = 0;
  if (tid == 0 && mytiles > 0) {
    load_x(0);
    x_pending = 1;
    x_par = 0;
  }
  // ---- W1^T as two bf16 terms (ranks past R zero), W2 (rows past R zero); W1 and W2
  // are contiguous fp32 arrays: every thread issues all its 16-byte loads at once
  {
    constexpr int NW1 = kMaxD * 16 / 4 / 256, NW2L = (16 * kMaxDK / 4 + 255) / 256;
    const int w14 = D * R / 4, w24 = R * dk / 4;
    float4 w1v[NW1], w2v[NW2L];
#pragma unroll
    for (int j = 0; j < NW1; ++j)
      if (tid + 256 * j < w14) w1v[j] = __ldg(reinterpret_cast<const float4*>(W1) + tid + 256 * j);
#pragma unroll
    for (int j = 0; j < NW2L; ++j)
      if (tid + 256 * j < w24) w2v[j] = __ldg(reinterpret_cast<const float4*>(W2) + tid + 256 * j);
    for (int i = tid; i < D * (16 - R); i += 256) {  // the zero ranks (none at R = 16)
      const int d = i / (16 - R), r = R + i % (16 - R);
      const uint32_t off = kmaj(d, r, 128u, 256u);
      *reinterpret_cast<__nv_bfloat16*>(sgen + lay.w1 + off) = __float2bfloat16_rn(0.f);
      *reinterpret_cast<__nv_bfloat16*>(sgen + lay.w1 + (uint32_t)(D / 8) * 256u + off) = __float2bfloat16_rn(0.f);
    }
    for (int i = tid; i < dk * (16 - R); i += 256) W2S[(i / (16 - R)) * 16 + R + i % (16 - R)] = 0.f;
#pragma unroll
    for (int j = 0; j < NW1; ++j) {
      const int q = tid + 256 * j;
      if (q < w14) {
        const float wv[4] = {w1v[j].x, w1v[j].y, w1v[j].z, w1v[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int idx = 4 * q + e, d = idx / R, r = idx - d * R;
          __nv_bfloat16 hi, lo;
          split_bf16(wv[e], hi, lo);
          const uint32_t off = kmaj(d, r, 128u, 256u);
          *reinterpret_cast<__nv_bfloat16*>(sgen + lay.w1 + off) = hi;
          *reinterpret_cast<__nv_bfloat16*>(sgen + lay.w1 + (uint32_t)(D / 8) * 256u + off) = lo;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < NW2L; ++j) {  // W2[r][k .. k + 3] -> W2^T[k .. k + 3][r]
      const int q = tid + 256 * j;
      if (q < w24) {
        const int r = (4 * q) / dk, k = 4 * q - r * dk;
        W2S[(k + 0) * 16 + r] = w2v[j].x;
        W2S[(k + 1) * 16 + r] = w2v[j].y;
        W2S[(k + 2) * 16 + r] = w2v[j].z;
        W2S[(k + 3) * 16 + r] = w2v[j].w;
      }
    }
  }
  for (int i = tid; i < kBM * 20; i += 256) US[i] = 0.f;  // ranks past R stay zero
  // dW2[r][lane] (r < 16) and db[lane]: this warp's sums over its 16 tokens of every
  // tile, added across the warps at the end
  float g2[16], gb = 0.f;  // lane k < d_k: dW2[r][k] for r = 0 .. 15 and db[k]
#pragma unroll
  for (int j = 0; j < 16; ++j) g2[j] = 0.f;
  const uint32_t tmem = sh.tmem;
  const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  uint8_t* stage = sgen + lay.stage + (uint32_t)warp * 4096u;  // this warp's dx staging: 32 rows x 128 bytes
  bool timed_out = false;

  // dz and u of a tile: its rows are contiguous in d log alpha, z and u, so every thread
  // issues all its 16-byte loads at once, one tile ahead (into registers)
  float4 la[NLD], lb[NLD], lc[2];
  auto issue_rows = [&](int i) {
    const long long r0 = tile_row(i);
    const int nr = (int)(rows - r0 < kBM ? rows - r0 : kBM);
    const int n4 = nr * dk / 4, u4 = nr * R / 4;  // d_k % 4 == 0, R % 4 == 0
#pragma unroll
    for (int j = 0; j < NLD; ++j)
      if (tid + 256 * j < n4) {
        la[j] = __ldg(reinterpret_cast<const float4*>(dla + r0 * dk) + tid + 256 * j);
        lb[j] = __ldg(reinterpret_cast<const float4*>(z + r0 * dk) + tid + 256 * j);
      }
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (tid + 256 * j < u4) lc[j] = __ldg(reinterpret_cast<const float4*>(u + r0 * R) + tid + 256 * j);
  };
  if (mytiles > 0) issue_rows(0);

  for (int i = 0; i < mytiles; ++i) {
    const long long row0 = tile_row(i);
    const int nrow = (int)(rows - row0 < kBM ? rows - row0 : kBM);
    // ---- dz = d log alpha * inv_tau * sigmoid(-z) and u into shared memory (rows past the end: zero)
    {
      const int n4 = nrow * dk / 4, u4 = nrow * R / 4;
      if (nrow < kBM) {  // the last, partial tile
        for (int idx = nrow * dk + tid; idx < kBM * dk; idx += 256) DZ[(idx / dk) * (dk + 1) + idx % dk] = 0.f;
        for (int idx = nrow * 16 + tid; idx < kBM * 16; idx += 256) US[(idx >> 4) * 20 + (idx & 15)] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < NLD; ++j) {
        const int q = tid + 256 * j;
        if (q < n4) {
          const float av[4] = {la[j].x, la[j].y, la[j].z, la[j].w}, bv[4] = {lb[j].x, lb[j].y, lb[j].z, lb[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = 4 * q + e, t = idx / dk;
            DZ[t * (dk + 1) + (idx - t * dk)] = av[e] * inv_tau * sigmoid_of_neg(bv[e]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int q = tid + 256 * j;
        if (q < u4) {
          const float cv[4] = {lc[j].x, lc[j].y, lc[j].z, lc[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = 4 * q + e, t = idx / R;
            US[t * 20 + (idx - t * R)] = cv[e];
          }
        }
      }
    }
    __syncthreads();
    // ---- du = dz W2^T: thread (token t, ranks 8 h .. 8 h + 7), as hi / lo terms in both layouts
    {
      const int t = tid & 127, h = tid >> 7;
      float du[8];
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) du[rr] = 0.f;
      for (int k = 0; k < dk; ++k) {
        const float d = DZ[t * (dk + 1) + k];
        const float4 w0 = *reinterpret_cast<const float4*>(W2S + k * 16 + 8 * h);
        const float4 w1 = *reinterpret_cast<const float4*>(W2S + k * 16 + 8 * h + 4);
        du[0] = fmaf(d, w0.x, du[0]); du[1] = fmaf(d, w0.y, du[1]);
        du[2] = fmaf(d, w0.z, du[2]); du[3] = fmaf(d, w0.w, du[3]);
        du[4] = fmaf(d, w1.x, du[4]); du[5] = fmaf(d, w1.y, du[5]);
        du[6] = fmaf(d, w1.z, du[6]); du[7] = fmaf(d, w1.w, du[7]);
      }
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int rr = 0; rr < 8; rr += 2) {
        __nv_bfloat16 h0, l0, h1, l1;
        split_bf16(du[rr], h0, l0);
        split_bf16(du[rr + 1], h1, l1);
        hw[rr / 2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        lw[rr / 2] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = 8 * h + rr + e;
          const uint32_t ob = kmaj(r, t, 128u, 2048u);
          *reinterpret_cast<__nv_bfloat16*>(sgen + lay.dub + ob) = e ? h1 : h0;
          *reinterpret_cast<__nv_bfloat16*>(sgen + lay.dub + 2u * 2048u + ob) = e ? l1 : l0;
        }
      }
      const uint32_t oa = kmaj(t, 8 * h, 128u, 256u);  // 8 consecutive ranks: one 16-byte core-matrix row
      *reinterpret_cast<uint4*>(sgen + lay.dua + oa) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sgen + lay.dua + 4096u + oa) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    // ---- dW2 += u^T dz and db += column sums of dz over this warp's 16 tokens (rows past
    // the end are zero); entry e = lane + 32 j: the lanes read one u value (broadcast) and
    // consecutive dz values of a row
    if (lane < dk) {
#pragma unroll 2
      for (int tt = 0; tt < 16; ++tt) {
        const int t = 16 * warp + tt;
        const float zk = DZ[t * (dk + 1) + lane];
        const float4* ur = reinterpret_cast<const float4*>(US + t * 20);  // the token's u (broadcast)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 u4 = ur[q];
          g2[4 * q] = fmaf(u4.x, zk, g2[4 * q]);
          g2[4 * q + 1] = fmaf(u4.y, zk, g2[4 * q + 1]);
          g2[4 * q + 2] = fmaf(u4.z, zk, g2[4 * q + 2]);
          g2[4 * q + 3] = fmaf(u4.w, zk, g2[4 * q + 3]);
        }
        gb += zk;
      }
    }
    fence_async_smem();  // du terms (and, first time, W1^T) are visible to the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- one thread: the x tile in, then dW1 += x^T [du_hi | du_lo] and dx = du W1^T
    if (tid == 0) {
      if (sh.abort || !mbar_wait(&sh.xfull, i & 1, kSpinLimitNs)) {
        sh.abort = 1;
        timed_out = true;
      } else {
        x_pending = 0;
        tc_fence_after();
        for (int mb = 0; mb < nmb; ++mb) {
#pragma unroll
          for (int ks = 0; ks < kBM / 16; ++ks) {
            uint64_t ad = sdesc_sw<128>(sb + lay.x + (uint32_t)(2 * mb) * kXB + 2048u * ks);
            ad &= ~(static_cast<uint64_t>(0x3FFF) << 16);  // leading byte offset: the next 64 channels' box
            ad |= static_cast<uint64_t>((kXB >> 4) & 0x3FFF) << 16;
            mma_bf16(tmem + kTmDW1 + 32u * mb, ad, sdesc(sb + lay.dub + 256u * ks, 128u, 2048u),
                     idesc_bf16(128, 32, true, false), (i > 0 || ks > 0) ? 1u : 0u);
          }
        }
        for (int hh = 0; hh < nh; ++hh)
#pragma unroll
          for (int tt = 0; tt < 4; ++tt) {
            const int ta = tt >> 1, tw = tt & 1;  // du term, W1 term
            mma_bf16(tmem + (uint32_t)(hh * NH), sdesc(sb + lay.dua + 4096u * ta, 128u, 256u),
                     sdesc(sb + lay.w1 + (uint32_t)tw * (D / 8) * 256u + (uint32_t)hh * (NH / 8) * 256u, 128u, 256u),
                     idesc_bf16(128, NH), tt ? 1u : 0u);
          }
        mma_commit(&sh.mma_done);
        mma_pending = 1;
        mma_par = i & 1;
      }
    }
    __syncthreads();  // sh.abort is uniform after this
    if (sh.abort) break;
    if (!mbar_wait(&sh.mma_done, i & 1, kSpinLimitNs)) timed_out = true;
    else if (tid == 0) mma_pending = 0;
    tc_fence_after();
    if (__syncthreads_or(timed_out)) {
      if (tid == 0) sh.abort = 1;
      break;
    }
    // the x tile and the du terms are consumed: the next tile's x comes in under the stores
    if (tid == 0 && i + 1 < mytiles) {
      load_x(i + 1);
      x_pending = 1;
      x_par = (i + 1) & 1;
    }
    if (i + 1 < mytiles) issue_rows(i + 1);  // they land while dx is written out
    // ---- dx rows: warp w reads TMEM lanes 32 (w % 4) .. (tokens) and half w / 4 of the
    // columns, 128 bytes of each row at a time; they pass through the warp's staging
    // (16-byte chunks swizzled by row) so that each store instruction writes whole
    // 128-byte lines of four (bf16) or eight (fp32) rows.
    {
      constexpr int CW = 128 / (int)sizeof(TOUT);  // columns per 128-byte piece of a row
      const int tq = 32 * (warp & 3);
      const int c_begin = (warp >> 2) * (D / 2), c_end = c_begin + D / 2;
      for (int c0 = c_begin; c0 < c_end; c0 += CW) {
        float v[CW];
        tmem_ld32(tmem + lane_base + (uint32_t)c0, v);
        if constexpr (CW == 64) tmem_ld32(tmem + lane_base + (uint32_t)c0 + 32u, v + 32);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // this lane's row, chunk c
          uint4 w;
          if constexpr (CW == 64)
            w = make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                           pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
          else
            w = make_uint4(__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]), __float_as_uint(v[4 * c + 2]),
                           __float_as_uint(v[4 * c + 3]));
          *reinterpret_cast<uint4*>(stage + lane * 128 + ((c ^ (lane & 7)) << 4)) = w;
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 8; ++it) {  // rows 4 it .. 4 it + 3, eight 16-byte chunks each
          const int row = 4 * it + (lane >> 3), c = lane & 7;
          const uint4 w = *reinterpret_cast<const uint4*>(stage + row * 128 + ((c ^ (row & 7)) << 4));
          if (tq + row < nrow)
            *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dx + (size_t)(row0 + tq + row) * D + c0) + 16 * c) = w;
        }
        __syncwarp();  // the staging is read before the next piece overwrites it
      }
    }
    tc_fence_before();  // TMEM reads precede the next tile's products (ordered by its barriers)
  }
  // ---- the CTA's partial sums (the abort flag's writer votes with its own view)
  const bool stopped = __syncthreads_or(sh.abort) != 0;
  if (mytiles > 0 && !stopped) {
    // every CTA adds the same addresses once, four ranks per 16-byte atomic; each starts at
    // another quad (and takes the channel blocks in another order) so that few CTAs meet
    // on one address at a time
    for (int m = 0; m < (nmb + 1) / 2; ++m) {
      const int mb = (warp >> 2) + 2 * ((m + (int)blockIdx.x) % ((nmb + 1) / 2));
      if (mb >= nmb) continue;
      float v[32];
      tmem_ld32(tmem + lane_base + kTmDW1 + 32u * mb, v);
      tmem_ld_wait();
      const int d = 128 * mb + 32 * (warp & 3) + lane;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const int r = 4 * ((qq + (int)blockIdx.x) & 3);
        if (r < R)
          atomicAdd(reinterpret_cast<float4*>(dW1 + (size_t)d * R + r),
                    make_float4(v[r] + v[16 + r], v[r + 1] + v[17 + r], v[r + 2] + v[18 + r], v[r + 3] + v[19 + r]));
      }
    }
  }
  if (mytiles > 0 && !stopped) {
    // dW2 and db: the eight warps' sums through shared memory (over the dz staging), then
    // one 16-byte atomic per quad
    float* red = DZ;  // [8][16 * d_k + d_k], over the dz and u staging (contiguous, 25 KB)
    const int ne = 16 * dk + dk;
    __syncthreads();  // every warp is done with the dz staging
    if (lane < dk) {
#pragma unroll
      for (int r = 0; r < 16; ++r) red[warp * ne + r * dk + lane] = g2[r];
      red[warp * ne + 16 * dk + lane] = gb;
    }
    __syncthreads();
    for (int q = tid; q < ne / 4; q += 256) {
      const int qr = (q + (int)blockIdx.x) % (ne / 4);  // rotated, as above
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float4 p = *reinterpret_cast<const float4*>(red + w * ne + 4 * qr);
        acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
      }
      const int e = 4 * qr;
      if (e < 16 * dk) {
        if (e / dk < R) atomicAdd(reinterpret_cast<float4*>(dW2 + e), acc);  // e = r d_k + k: dW2 is [R][d_k]
      } else if (db != nullptr) {
        atomicAdd(reinterpret_cast<float4*>(db + (e - 16 * dk)), acc);
      }
    }
  }
  // ---- drain: a requested x tile and the last products complete before the CTA exits
  if (tid == 0) {
    if (x_pending) mbar_wait(&sh.xfull, x_par, kSpinLimitNs);
    if (mma_pending) mbar_wait(&sh.mma_done, mma_par, kSpinLimitNs);
  }
  if (sh.abort && status != nullptr && tid == 0) set_status(status, DIG_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

bool gate_proj_bwd_tc_eligible(long long rows, int D, int R, int dk, int tin) {
  return tin == DIG_BF16 && rows > 0 && rows <= 0x7FFFFFFFLL && R >= 1 && R <= 16 && R % 4 == 0 && D % 128 == 0 &&
         D <= kMaxD && dk >= 4 && dk <= kMaxDK && dk % 4 == 0 && tmap_available();
}

// dW1, dW2 and db must be zero on the stream already.  `launched` stays false
// when the tensor map cannot be encoded (the caller runs the CUDA-core kernel).
cudaError_t launch_gate_proj_bwd_tc(const void* x, const float* W1, const float* W2, const float* u, const float* z,
                                    const float* dla, float inv_tau, void* dx, float* dW1, float* dW2, float* db,
                                    long long rows, int D, int R, int dk, int tout, uint32_t* status, cudaStream_t s,
                                    bool* launched) {
  *launched = false;
  CUtensorMap m;
  memset(&m, 0, sizeof(m));
  if (!tmap_rows(&m, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, (uint64_t)rows, kKB, kBM, 128)) return cudaSuccess;
  // at least 116 KB, so that one CTA fits per SM: each takes all 512 TMEM columns
  const uint32_t smem = GbLayout(D, dk).total + 1024 > 116u * 1024u ? GbLayout(D, dk).total + 1024 : 116u * 1024u;
  const long long ntiles = (rows + kBM - 1) / kBM;
  const int grid = (int)(ntiles < num_sms() ? ntiles : num_sms());
  cudaError_t e;
  if (tout == DIG_BF16) {
    auto k = gate_proj_bwd_tc_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = launch_pdl(k, dim3(grid), dim3(256), smem, s, m, W1, W2, u, z, dla, inv_tau,
                     static_cast<__nv_bfloat16*>(dx), dW1, dW2, db, rows, D, R, dk, status);
  } else {
    auto k = gate_proj_bwd_tc_kernel<float>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = launch_pdl(k, dim3(grid), dim3(256), smem, s, m, W1, W2, u, z, dla, inv_tau, static_cast<float*>(dx), dW1,
                     dW2, db, rows, D, R, dk, status);
  }
  if (e == cudaSuccess) *launched = true;
  return e;
}

}  // namespace dig
