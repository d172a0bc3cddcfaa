// gla_gate.cu -- per-chunk gate factors shared by every head.
//
// For each (batch, gate head, chunk of C scan positions) this computes, from the
// gate logits z (DiG slides, GLA eq. (5): alpha = sigmoid(z)^(1/tau)):
//   b_t   = sum of log2(alpha) over the chunk's tokens up to t (inclusive)
//   r     = b at the chunk's middle token C/2 - 1   (factorisation reference)
//   Gamma = b at the chunk's last token             (chunk decay)
// and stores, in scan order,
//   EQ[t][c] = 2^(b_t - r)                                            per token
//   CH[chunk] = { 2^r, 2^(Gamma - r), 2^Gamma, Gamma }[c]             per chunk
// The GLA forward and backward kernels read these instead of recomputing the
// gate for every head.  A chunk whose |b - r| exceeds 115 (2^115 ~ e^80) in some
// channel is outside the range the factorisation covers: DIG_ERR_GATE_RANGE.
#include "gla.h"
#include "gla_common.cuh"

namespace dig {

template <int C, int DK>
__global__ void __launch_bounds__(C) gla_gate_kernel(const GlaArgs a, int nchunks, float* __restrict__ EQ,
                                                     float* __restrict__ CH) {
  constexpr int NW = C / 32;
  __shared__ float s_tot[NW][DK];
  __shared__ float s_ref[DK];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int n = blockIdx.x;
  const int bz = blockIdx.y;  // b * gate_heads + hz
  const int b = bz / a.gate_heads, hz = bz - b * a.gate_heads;
  const int p = n * C + t;
  const bool valid = p < a.L;
  float b2[DK];
  if (valid) {
    const int g = scan_to_grid(p, a.L, a.Hg, a.Wg, a.mode);
    const float4* zp = reinterpret_cast<const float4*>(a.z + (((size_t)b * a.L + g) * a.gate_heads + hz) * DK);
#pragma unroll
    for (int i = 0; i < DK / 4; ++i) {
      const float4 u = __ldg(zp + i);
      b2[4 * i + 0] = log2_decay(u.x, a.inv_tau);
      b2[4 * i + 1] = log2_decay(u.y, a.inv_tau);
      b2[4 * i + 2] = log2_decay(u.z, a.inv_tau);
      b2[4 * i + 3] = log2_decay(u.w, a.inv_tau);
    }
  } else {
#pragma unroll
    for (int i = 0; i < DK; ++i) b2[i] = 0.f;  // padding tokens do not decay
  }
#pragma unroll
  for (int i = 0; i < DK; ++i) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, b2[i], off);
      if (lane >= off) b2[i] += y;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int i = 0; i < DK; ++i) s_tot[warp][i] = b2[i];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < DK; ++i) {
    float pre = 0.f;
#pragma unroll
    for (int u = 0; u < NW; ++u) pre += (u < warp) ? s_tot[u][i] : 0.f;
    b2[i] += pre;
  }
  if (t == C / 2 - 1) {
#pragma unroll
    for (int i = 0; i < DK; ++i) s_ref[i] = b2[i];
  }
  __syncthreads();
  bool bad = false;
  if (valid) {
    float4* eq = reinterpret_cast<float4*>(EQ + ((size_t)bz * a.L + p) * DK);
#pragma unroll
    for (int i = 0; i < DK / 4; ++i) {
      float d[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        d[u] = b2[4 * i + u] - s_ref[4 * i + u];
        bad |= fabsf(d[u]) > 115.f;
      }
      eq[i] = make_float4(exp2f(d[0]), exp2f(d[1]), exp2f(d[2]), exp2f(d[3]));
    }
  }
  if (bad) set_status(a.status, DIG_ERR_GATE_RANGE);
  if (t < DK) {
    float gam = 0.f;
#pragma unroll
    for (int u = 0; u < NW; ++u) gam += s_tot[u][t];
    const float r = s_ref[t];
    float* ch = CH + ((size_t)bz * nchunks + n) * 4 * DK;
    ch[0 * DK + t] = exp2f(r);
    ch[1 * DK + t] = exp2f(gam - r);
    ch[2 * DK + t] = exp2f(gam);
    ch[3 * DK + t] = gam;
  }
}

template <int C>
static cudaError_t gate_dispatch(const GlaArgs& a, int dk, int nchunks, float* EQ, float* CH,
                                 cudaStream_t s) {
  const dim3 grid(nchunks, a.B * a.gate_heads);
  switch (dk) {
    case 32: gla_gate_kernel<C, 32><<<grid, C, 0, s>>>(a, nchunks, EQ, CH); break;
    case 36: gla_gate_kernel<C, 36><<<grid, C, 0, s>>>(a, nchunks, EQ, CH); break;
    case 64: gla_gate_kernel<C, 64><<<grid, C, 0, s>>>(a, nchunks, EQ, CH); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_gla_gate(const GlaArgs& a, int chunk, int dk, int nchunks, float* EQ, float* CH,
                            cudaStream_t s) {
  if (nchunks > 2147483647 || a.B * a.gate_heads > 65535) return cudaErrorInvalidValue;
  switch (chunk) {
    case 128: return gate_dispatch<128>(a, dk, nchunks, EQ, CH, s);
    case 64: return gate_dispatch<64>(a, dk, nchunks, EQ, CH, s);
    case 32: return gate_dispatch<32>(a, dk, nchunks, EQ, CH, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dig
