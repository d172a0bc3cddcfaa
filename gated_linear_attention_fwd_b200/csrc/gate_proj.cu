// gate_proj.cu -- the gate logits' low-rank projection and its backward (DiG
// slides, "Gated Linear Attention Transformer (GLA) の導入", eq. (5): the gate is
// sigmoid of a projection of the block input, made low-rank D -> R -> d_k):
//
//   u = x W1   [rows, R],   z = u W2 + b   [rows, d_k]
//
// and, from the GLA backward's d log(alpha) with log(alpha) = inv_tau logsigmoid(z):
//
//   dz = dla inv_tau sigmoid(-z),  du = dz W2^T,  dx = du W1^T,
//   dW1 = x^T du,  dW2 = u^T dz,  db = sum_rows dz.
//
// About 2 D R multiply-adds per token against 2 D bytes of x (bf16): HBM-scale
// work, kept on the FP32 pipes.  Tiles of 64 tokens; the weights stay in shared
// memory for the whole (persistent) block.
#include "dig_common.cuh"
#include "gate_proj.h"
#include "gla_common.cuh"

namespace dig {

namespace {

constexpr int kTT = 64;  // tokens per tile
constexpr int kXB = 8;   // forward: 8-value vectors of x loaded ahead per thread
constexpr int kXT = 16;  // backward dW1: tokens of x loaded ahead per thread

// 8 consecutive values of a row as fp32 (one 16-byte load for bf16, two for fp32)
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* v) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float* v) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}

// Copies a weight matrix into shared memory in the layout `dst[i] = src_at(i)` (0
// where src_at returns a negative index), i < n, with 8 loads in flight per
// thread: the copy costs a few memory round trips instead of one per element.
template <typename F>
__device__ __forceinline__ void stage_weights(float* dst, const float* __restrict__ src, int n, F src_at) {
  for (int i0 = threadIdx.x; i0 < n; i0 += 8 * blockDim.x) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      const long long j = i < n ? src_at(i) : -1;
      v[u] = j >= 0 ? __ldg(src + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < n) dst[i] = v[u];
    }
  }
}

__device__ __forceinline__ float sigmoid_neg(float z) {  // sigmoid(-z)
  return __fdividef(1.f, 1.f + ex2(z * kLog2e));
}

}  // namespace

// Dynamic shared memory of the forward, in bytes: fp32 W1 [D][RT] (columns >= R
// zero), W2 [RT][dk] (rows >= R zero) and u [kTT][RT + 1].
inline size_t gate_fwd_smem(int D, int RT, int dk) {
  return 4 * ((size_t)D * RT + (size_t)RT * dk + (size_t)kTT * (RT + 1));
}

// Forward.  Thread (token t = tid / 4, quarter g = tid % 4) forms RQ = RT / 4 of
// the token's u values, walking x's row in 8-value vectors against W1's rows in
// shared memory; then the block forms z (and writes u) from u in shared memory,
// one coalesced output per thread and step.
template <typename TIN, int RT>
__global__ void __launch_bounds__(256) gate_proj_fwd_kernel(const TIN* __restrict__ x, const float* __restrict__ W1,
                                                            const float* __restrict__ W2,
                                                            const float* __restrict__ b, float* __restrict__ z,
                                                            float* __restrict__ u, long long rows, int D, int R,
                                                            int dk) {
  constexpr int RQ = RT / 4;
  extern __shared__ __align__(16) float gp_smem[];
  float* W1s = gp_smem;                         // [D][RT]
  float* W2s = W1s + (size_t)D * RT;            // [RT][dk]
  float* us = W2s + (size_t)RT * dk;            // [kTT][RT + 1]
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  stage_weights(W1s, W1, D * RT, [&](int i) -> long long {
    const int d = i / RT, r = i % RT;
    return r < R ? (long long)d * R + r : -1;
  });
  stage_weights(W2s, W2, RT * dk, [&](int i) -> long long {
    const int r = i / dk, k = i % dk;
    return r < R ? (long long)r * dk + k : -1;
  });
  __syncthreads();
  const int tl = threadIdx.x >> 2, g = threadIdx.x & 3;
  const long long ntiles = (rows + kTT - 1) / kTT;
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const long long row0 = tile * kTT;
    const long long row = row0 + tl;
    float acc[RQ];
#pragma unroll
    for (int j = 0; j < RQ; ++j) acc[j] = 0.f;
    if (row < rows) {
      const TIN* xr = x + (size_t)row * D;
      // kXB vectors of x in flight per thread before their products
      for (int c0 = 0; c0 < D; c0 += 8 * kXB) {
        float xv[kXB][8];
#pragma unroll
        for (int q = 0; q < kXB; ++q)
          if (c0 + 8 * q < D) load8(xr + c0 + 8 * q, xv[q]);
#pragma unroll
        for (int q = 0; q < kXB; ++q) {
          if (c0 + 8 * q >= D) break;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float* wrow = W1s + (size_t)(c0 + 8 * q + e) * RT + g * RQ;
#pragma unroll
            for (int j = 0; j < RQ; j += 4) {
              const float4 wv = *reinterpret_cast<const float4*>(wrow + j);
              acc[j] = fmaf(xv[q][e], wv.x, acc[j]);
              acc[j + 1] = fmaf(xv[q][e], wv.y, acc[j + 1]);
              acc[j + 2] = fmaf(xv[q][e], wv.z, acc[j + 2]);
              acc[j + 3] = fmaf(xv[q][e], wv.w, acc[j + 3]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < RQ; ++j) us[tl * (RT + 1) + g * RQ + j] = acc[j];
    __syncthreads();
    const int nt = (int)(rows - row0 < kTT ? rows - row0 : kTT);
    for (int i = threadIdx.x; i < nt * dk; i += blockDim.x) {
      const int t = i / dk, k = i % dk;
      float v = b ? __ldg(b + k) : 0.f;
#pragma unroll 8
      for (int r = 0; r < RT; ++r) v = fmaf(us[t * (RT + 1) + r], W2s[r * dk + k], v);
      z[(size_t)(row0 + t) * dk + k] = v;
    }
    if (u)
      for (int i = threadIdx.x; i < nt * R; i += blockDim.x) {
        const int t = i / R, r = i % R;
        u[(size_t)(row0 + t) * R + r] = us[t * (RT + 1) + r];
      }
    __syncthreads();  // us is rewritten by the next tile
  }
}

// Dynamic shared memory of the backward, in bytes: fp32 W1^T [RT][D], dW1^T
// partials [RT][D], W2^T [dk][RT], dz [kTT][dk + 1], u and du [kTT][RT + 4] each
// (rows of u and du start on 16-byte boundaries).
inline size_t gate_bwd_smem(int D, int RT, int dk) {
  return 4 * (2 * (size_t)RT * D + (size_t)dk * RT + (size_t)kTT * (dk + 1) + 2 * (size_t)kTT * (RT + 4));
}

__device__ __forceinline__ void store2(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
}
__device__ __forceinline__ void store2(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}

// Backward.  Per tile of 64 tokens: dz (from d log alpha and z) and u into shared
// memory; du = dz W2^T; the dW2 and db partials (each thread owns fixed (r, k)
// entries, in registers); dx = du W1^T, two consecutive columns of one token per
// thread and step (consecutive threads on consecutive columns: coalesced stores,
// conflict-free reads of W1^T); the dW1 partials, each thread owning whole
// columns d of dW1^T in shared memory (x read once, consecutive threads on
// consecutive d).  At the end every block adds its partials to dW1, dW2 and db
// with atomics.
template <typename TIN, typename TOUT, int RT, int DKMAX>
__global__ void __launch_bounds__(256) gate_proj_bwd_kernel(const TIN* __restrict__ x, const float* __restrict__ W1,
                                                            const float* __restrict__ W2,
                                                            const float* __restrict__ uin,
                                                            const float* __restrict__ z,
                                                            const float* __restrict__ dla, float inv_tau,
                                                            TOUT* __restrict__ dx, float* __restrict__ dW1,
                                                            float* __restrict__ dW2, float* __restrict__ db,
                                                            long long rows, int D, int R, int dk) {
  constexpr int NW2 = (RT * DKMAX + 255) / 256;  // dW2 entries per thread
  constexpr int UP = RT + 4;                     // row pitch of u and du
  extern __shared__ __align__(16) float gp_smem[];
  float* W1T = gp_smem;                        // [RT][D]
  float* G1T = W1T + (size_t)RT * D;           // [RT][D] dW1^T partials
  float* W2T = G1T + (size_t)RT * D;           // [dk][RT]
  float* dzs = W2T + (size_t)dk * RT;          // [kTT][dk + 1]
  float* us = dzs + (size_t)kTT * (dk + 1);    // [kTT][UP]
  float* dus = us + (size_t)kTT * UP;          // [kTT][UP]
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  stage_weights(W1T, W1, RT * D, [&](int i) -> long long {
    const int r = i / D, d = i % D;
    return r < R ? (long long)d * R + r : -1;
  });
  for (int i = threadIdx.x; i < RT * D; i += blockDim.x) G1T[i] = 0.f;
  stage_weights(W2T, W2, dk * RT, [&](int i) -> long long {
    const int k = i / RT, r = i % RT;
    return r < R ? (long long)r * dk + k : -1;
  });
  float g2[NW2], gb = 0.f;
#pragma unroll
  for (int j = 0; j < NW2; ++j) g2[j] = 0.f;
  __syncthreads();
  const int npair = D / 2;
  const long long ntiles = (rows + kTT - 1) / kTT;
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const long long row0 = tile * kTT;
    const int nt = (int)(rows - row0 < kTT ? rows - row0 : kTT);
    for (int i = threadIdx.x; i < kTT * dk; i += blockDim.x) {
      const int t = i / dk, k = i % dk;
      float v = 0.f;
      if (t < nt) {
        const size_t o = (size_t)(row0 + t) * dk + k;
        v = __ldg(dla + o) * inv_tau * sigmoid_neg(__ldg(z + o));
      }
      dzs[t * (dk + 1) + k] = v;
    }
    for (int i = threadIdx.x; i < kTT * RT; i += blockDim.x) {
      const int t = i / RT, r = i % RT;
      us[t * UP + r] = (t < nt && r < R) ? __ldg(uin + (size_t)(row0 + t) * R + r) : 0.f;
    }
    __syncthreads();
    // du = dz W2^T
    for (int i = threadIdx.x; i < kTT * RT; i += blockDim.x) {
      const int t = i / RT, r = i % RT;
      float v = 0.f;
      for (int k = 0; k < dk; ++k) v = fmaf(dzs[t * (dk + 1) + k], W2T[k * RT + r], v);
      dus[t * UP + r] = v;
    }
    // dW2 = u^T dz and db = sum dz (fixed entries per thread)
#pragma unroll
    for (int j = 0; j < NW2; ++j) {
      const int e = threadIdx.x + 256 * j;
      if (e < RT * dk) {
        const int r = e / dk, k = e % dk;
        float v = 0.f;
        for (int t = 0; t < nt; ++t) v = fmaf(us[t * UP + r], dzs[t * (dk + 1) + k], v);
        g2[j] += v;
      }
    }
    if (threadIdx.x < dk)
      for (int t = 0; t < nt; ++t) gb += dzs[t * (dk + 1) + threadIdx.x];
    __syncthreads();  // du complete
    // dx = du W1^T
    for (int i = threadIdx.x; i < nt * npair; i += blockDim.x) {
      const int t = i / npair, d0 = 2 * (i % npair);
      float v0 = 0.f, v1 = 0.f;
#pragma unroll 4
      for (int r = 0; r < RT; ++r) {
        const float g = dus[t * UP + r];
        const float2 wv = *reinterpret_cast<const float2*>(W1T + (size_t)r * D + d0);
        v0 = fmaf(g, wv.x, v0);
        v1 = fmaf(g, wv.y, v1);
      }
      store2(dx + (size_t)(row0 + t) * D + d0, v0, v1);
    }
    // dW1^T += du^T x: thread owns columns d = tid, tid + 256, ...
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float a[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) a[r] = 0.f;
      // kXT tokens of x in flight per thread; du rows at and past nt are zero
      for (int t0 = 0; t0 < nt; t0 += kXT) {
        float xv[kXT];
#pragma unroll
        for (int j = 0; j < kXT; ++j)
          xv[j] = t0 + j < nt ? static_cast<float>(x[(size_t)(row0 + t0 + j) * D + d]) : 0.f;
#pragma unroll
        for (int j = 0; j < kXT; ++j) {
#pragma unroll
          for (int r = 0; r < RT; r += 4) {
            const float4 g4 = *reinterpret_cast<const float4*>(dus + (t0 + j) * UP + r);
            a[r] = fmaf(xv[j], g4.x, a[r]);
            a[r + 1] = fmaf(xv[j], g4.y, a[r + 1]);
            a[r + 2] = fmaf(xv[j], g4.z, a[r + 2]);
            a[r + 3] = fmaf(xv[j], g4.w, a[r + 3]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RT; ++r) G1T[(size_t)r * D + d] += a[r];
    }
    __syncthreads();  // dzs, us, dus are rewritten by the next tile
  }
  for (int i = threadIdx.x; i < D * R; i += blockDim.x) {
    const int d = i / R, r = i % R;
    atomicAdd(dW1 + i, G1T[(size_t)r * D + d]);
  }
#pragma unroll
  for (int j = 0; j < NW2; ++j) {
    const int e = threadIdx.x + 256 * j;
    if (e < RT * dk) {
      const int r = e / dk, k = e % dk;
      if (r < R) atomicAdd(dW2 + (size_t)r * dk + k, g2[j]);
    }
  }
  if (db && threadIdx.x < dk) atomicAdd(db + threadIdx.x, gb);
}

namespace {

// a[0 .. na), b[0 .. nb), c[0 .. nc) = 0
__global__ void __launch_bounds__(256) zero3_kernel(float* a, int na, float* b, int nb, float* c, int nc) {
  griddep_wait();  // the kernels before this one have completed (they may read the buffers)
  griddep_launch_dependents();
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i < na) a[i] = 0.f;
  else if (i < na + nb) b[i - na] = 0.f;
  else if (i < na + nb + nc) c[i - na - nb] = 0.f;
}

int resident_grid(const void* kern, size_t smem, long long work, int cap_per_sm) {
  int dev = 0, sms = 148, per_sm = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  if (per_sm > cap_per_sm) per_sm = cap_per_sm;
  const long long g = (long long)sms * per_sm;
  return (int)(work < g ? work : g);
}

template <typename TIN, int RT>
cudaError_t fwd_typed(const void* x, const float* W1, const float* W2, const float* b, float* z, float* u,
                      long long rows, int D, int R, int dk, cudaStream_t s) {
  auto kern = gate_proj_fwd_kernel<TIN, RT>;
  const size_t smem = gate_fwd_smem(D, RT, dk);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = resident_grid(reinterpret_cast<const void*>(kern), smem, (rows + kTT - 1) / kTT, 8);
  return launch_pdl(kern, dim3(grid), dim3(256), smem, s, reinterpret_cast<const TIN*>(x), W1, W2, b, z, u, rows,
                    D, R, dk);
}

template <typename TIN, typename TOUT, int RT>
cudaError_t bwd_typed(const void* x, const float* W1, const float* W2, const float* u, const float* z,
                      const float* dla, float inv_tau, void* dx, float* dW1, float* dW2, float* db, long long rows,
                      int D, int R, int dk, cudaStream_t s) {
  auto kern = gate_proj_bwd_kernel<TIN, TOUT, RT, 128>;
  const size_t smem = gate_bwd_smem(D, RT, dk);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // each block adds D*R + R*dk + dk atomics at its end: keep to one wave of at most 2 per SM
  const int grid = resident_grid(reinterpret_cast<const void*>(kern), smem, (rows + kTT - 1) / kTT, 2);
  return launch_pdl(kern, dim3(grid), dim3(256), smem, s, reinterpret_cast<const TIN*>(x), W1, W2, u, z, dla,
                    inv_tau, reinterpret_cast<TOUT*>(dx), dW1, dW2, db, rows, D, R, dk);
}

}  // namespace

size_t gate_proj_smem_bytes(int D, int R, int dk, bool backward) {
  const int RT = R <= 16 ? 16 : 32;
  return backward ? gate_bwd_smem(D, RT, dk) : gate_fwd_smem(D, RT, dk);
}

bool gate_proj_tc_eligible(long long rows, int D, int R, int dk, int tin);  // gate_proj_tc.cu
cudaError_t launch_gate_proj_tc(const void* x, const float* W1, const float* W2, const float* b, float* z, float* u,
                                long long rows, int D, int R, int dk, uint32_t* status, cudaStream_t s,
                                bool* launched);

cudaError_t launch_gate_proj_fwd(const void* x, const float* W1, const float* W2, const float* b, float* z, float* u,
                                 long long rows, int D, int R, int dk, int tin, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (rows == 0) return cudaSuccess;
  if (gate_proj_tc_eligible(rows, D, R, dk, tin)) {  // bf16 x: x W1 on the tensor cores
    bool launched = false;
    const cudaError_t e = launch_gate_proj_tc(x, W1, W2, b, z, u, rows, D, R, dk, nullptr, s, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  if (R <= 16)
    return tin == DIG_BF16 ? fwd_typed<bf, 16>(x, W1, W2, b, z, u, rows, D, R, dk, s)
                           : fwd_typed<float, 16>(x, W1, W2, b, z, u, rows, D, R, dk, s);
  return tin == DIG_BF16 ? fwd_typed<bf, 32>(x, W1, W2, b, z, u, rows, D, R, dk, s)
                         : fwd_typed<float, 32>(x, W1, W2, b, z, u, rows, D, R, dk, s);
}

bool gate_proj_bwd_tc_eligible(long long rows, int D, int R, int dk, int tin);  // gate_proj_bwd_tc.cu
cudaError_t launch_gate_proj_bwd_tc(const void* x, const float* W1, const float* W2, const float* u, const float* z,
                                    const float* dla, float inv_tau, void* dx, float* dW1, float* dW2, float* db,
                                    long long rows, int D, int R, int dk, int tout, uint32_t* status, cudaStream_t s,
                                    bool* launched);

cudaError_t launch_gate_proj_bwd(const void* x, const float* W1, const float* W2, const float* u, const float* z,
                                 const float* dla, float inv_tau, void* dx, float* dW1, float* dW2, float* db,
                                 long long rows, int D, int R, int dk, int tin, int tout, cudaStream_t s) {
  using bf = __nv_bfloat16;
  // the weight gradients are sums of the blocks' atomics: zeroed first, by one kernel in
  // the stream's dependent-launch chain
  const int nw1 = D * R, nw2 = R * dk, nb = db ? dk : 0;
  cudaError_t e = launch_pdl(zero3_kernel, dim3((nw1 + nw2 + nb + 255) / 256), dim3(256), 0, s, dW1, nw1, dW2, nw2,
                             db, nb);
  if (e != cudaSuccess || rows == 0) return e;
  if (gate_proj_bwd_tc_eligible(rows, D, R, dk, tin)) {  // bf16 x: dx and dW1 on the tensor cores
    bool launched = false;
    e = launch_gate_proj_bwd_tc(x, W1, W2, u, z, dla, inv_tau, dx, dW1, dW2, db, rows, D, R, dk, tout, nullptr, s,
                                &launched);
    if (e != cudaSuccess || launched) return e;
  }
#define DIG_GATE_BWD(TI, TO, RT) bwd_typed<TI, TO, RT>(x, W1, W2, u, z, dla, inv_tau, dx, dW1, dW2, db, rows, D, R, dk, s)
  if (R <= 16) {
    if (tin == DIG_BF16) return tout == DIG_BF16 ? DIG_GATE_BWD(bf, bf, 16) : DIG_GATE_BWD(bf, float, 16);
    return tout == DIG_BF16 ? DIG_GATE_BWD(float, bf, 16) : DIG_GATE_BWD(float, float, 16);
  }
  if (tin == DIG_BF16) return tout == DIG_BF16 ? DIG_GATE_BWD(bf, bf, 32) : DIG_GATE_BWD(bf, float, 32);
  return tout == DIG_BF16 ? DIG_GATE_BWD(float, bf, 32) : DIG_GATE_BWD(float, float, 32);
#undef DIG_GATE_BWD
}

}  // namespace dig
