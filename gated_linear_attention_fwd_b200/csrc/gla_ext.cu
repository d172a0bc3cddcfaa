// gla_ext.cu -- the pieces of the extended GLA entry points (value gate and
// state input / output; DiG slides, "Gated Linear Attention Transformer (GLA)
// の導入", eq. (5): G_t = alpha_t^T beta_t, S_t = G_t (*) S_{t-1} + k_t^T v_t)
// that the chunk kernels do not cover:
//   * widening bf16 inputs to fp32 (the extended path runs the fp32 kernels);
//   * d log beta.  With e the natural-log cumsum of log beta over a chunk, the
//     loss depends on e_u through o_u = (...) e^{e_u} and through the decays
//     e^{-e_u} of v_u; so dL/de_u = dO_u o_u - v_u dv_u per value channel, and
//     e_u enters every later token of the chunk and, through the chunk's total,
//     the state leaving it: d log beta_t = sum_{u >= t in chunk} (dO_u o_u -
//     v_u dv_u) + sum_c (S_{n+1} (*) G_n)[c][:] (G_n the gradient of S_{n+1}).
#include "gla_chunk.cuh"

namespace dig {

namespace {

__global__ void __launch_bounds__(256) widen_bf16_kernel(const __nv_bfloat16* __restrict__ src, float* __restrict__ dst,
                                                         long long n8) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src) + i);
    float4* d = reinterpret_cast<float4*>(dst) + 2 * i;
    d[0] = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xFFFF0000u));
    d[1] = make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xFFFF0000u), __uint_as_float(u.w << 16),
                       __uint_as_float(u.w & 0xFFFF0000u));
  }
}

__device__ __forceinline__ float ld_any(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_any(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// One block per (sequence, chunk) unit: the chunk's tokens' terms dO o - v dv per
// value channel, their suffix sums in scan order, plus the boundary term; added
// (heads sharing the gate) or written into d log beta [B, L, gate_heads, DV].
template <typename TOUT, int C, int DV>
__global__ void __launch_bounds__(256) gla_dlogbeta_kernel(const GlaArgs a, const TOUT* __restrict__ o,
                                                           float* __restrict__ dlb, int DK) {
  constexpr int NSG = 256 / DV, SEGL = cdiv(C, NSG);
  __shared__ float X[C][DV + 1];
  __shared__ float bnd[DV];
  __shared__ float segtot[8][DV];
  __shared__ long long grows[C];
  griddep_wait();
  griddep_launch_dependents();
  const int tid = threadIdx.x;
  const int nunits = a.B * a.H * a.nchunks;
  const float* v = static_cast<const float*>(a.v);
  const float* dO = static_cast<const float*>(a.dO);
  const TOUT* dv = static_cast<const TOUT*>(a.dv);
  for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
    const Unit U(a, u);
    const int hz = U.bz - U.b * a.gate_heads;
    if (tid < C) {
      const int p = U.n * C + tid;
      grows[tid] = p < a.L ? (long long)U.b * a.L + scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode) : -1;
    }
    if (tid < DV) {  // sum_c S_{n+1}[j][c] G_n[j][c] (the state after the last chunk for the last one)
      const float* s1 = U.n + 1 < a.nchunks ? a.dsn + (size_t)(u + 1) * DV * DK : a.sfin + (size_t)U.bh * DV * DK;
      const float* g = a.dhn + (size_t)u * DV * DK;
      float acc = 0.f;
      for (int c = 0; c < DK; ++c) acc = fmaf(__ldcg(s1 + (size_t)tid * DK + c), __ldcg(g + (size_t)tid * DK + c), acc);
      bnd[tid] = acc;
    }
    __syncthreads();
    for (int i = tid; i < C * DV; i += 256) {
      const int t = i / DV, j = i - t * DV;
      const long long gr = grows[t];
      float x = 0.f;
      if (gr >= 0) {
        const size_t off = ((size_t)gr * a.H + U.h) * DV + j;
        x = __ldg(dO + off) * ld_any(o + off) - __ldg(v + off) * ld_any(dv + off);
      }
      X[t][j] = x;
    }
    __syncthreads();
    const int j = tid % DV, sg = tid / DV;
    const int t0 = sg * SEGL, t1 = min(C, t0 + SEGL);
    if (sg < NSG) {
      float acc = 0.f;
      for (int t = t1 - 1; t >= t0; --t) {
        acc += X[t][j];
        X[t][j] = acc;
      }
      segtot[sg][j] = acc;
    }
    __syncthreads();
    if (sg < NSG) {
      float post = bnd[j];
      for (int s2 = sg + 1; s2 < NSG; ++s2) post += segtot[s2][j];
      for (int t = t0; t < t1; ++t) {
        const long long gr = grows[t];
        if (gr >= 0) {
          float* dst = dlb + ((size_t)gr * a.gate_heads + hz) * DV + j;
          if (a.gate_heads == 1) atomicAdd(dst, X[t][j] + post);
          else *dst = X[t][j] + post;
        }
      }
    }
    __syncthreads();  // the token table, X and the totals are reused by the next unit
  }
}

}  // namespace

cudaError_t launch_widen_bf16(const void* src, float* dst, long long n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (n % 8 != 0) return cudaErrorInvalidValue;
  const long long n8 = n / 8;
  const long long want = (n8 + 255) / 256;
  const int grid = (int)(want < 148LL * 8 ? want : 148LL * 8);
  return launch_pdl(widen_bf16_kernel, dim3(grid), dim3(256), 0, s, static_cast<const __nv_bfloat16*>(src), dst,
                    n8);
}

// d log beta (zeroed first when heads share the gate); `o` is the forward's output
// in the output type, dv the gradient just written (same type); v and dO of `a`
// are fp32.
cudaError_t launch_dlogbeta(const GlaArgs& a, int dk, int dv, int tout, const void* o, float* dlb, cudaStream_t s) {
  const long long units = (long long)a.B * a.H * a.nchunks;
  if (units <= 0) return cudaSuccess;
  if (a.gate_heads == 1) {
    const cudaError_t e = cudaMemsetAsync(dlb, 0, (size_t)a.B * a.L * dv * sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  const int grid = persistent_grid(4, units);
  constexpr int C = 64;
#define DIG_DLB(TO, DV)                                                                                              \
  launch_pdl(gla_dlogbeta_kernel<TO, C, DV>, dim3(grid), dim3(256), 0, s, a, static_cast<const TO*>(o), dlb, dk)
  if (dv == 64) return tout == DIG_BF16 ? DIG_DLB(__nv_bfloat16, 64) : DIG_DLB(float, 64);
  if (dv == 72) return tout == DIG_BF16 ? DIG_DLB(__nv_bfloat16, 72) : DIG_DLB(float, 72);
#undef DIG_DLB
  return cudaErrorInvalidValue;
}

}  // namespace dig
