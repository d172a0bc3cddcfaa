// dig_block.cu -- the element-wise steps of a DiG block around its GLA token
// mixer (DiG slides, Fig. 4 and the "DiG Block" section): adaptive RMS
// normalisation with the scale / shift regressed from the conditioning, the
// gated residual adds, and the activations of the conditioning MLP (SiLU) and
// of the feed-forward network (GELU).  The block's dense projections are plain
// library GEMMs; these kernels are the rest of it.  All are memory-bound: one
// read and one write per element, 16-byte accesses, grid-stride loops.
#include <cuda_bf16.h>

#include "../../include/dig.h"
#include "dig_common.cuh"
#include "gla_common.cuh"

namespace dig {

void set_last_error(const char* msg);  // dig_api.cu

namespace {

__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void st8(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// One warp per row of D values (D % 256 == 0 or any multiple of 8 up to 8 * 32 * 8):
// y = x / sqrt(mean(x^2) + eps) * (1 + scale[b]) + shift[b].
__global__ void __launch_bounds__(256) rmsnorm_mod_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const float* __restrict__ shift,
                                                          const float* __restrict__ scale, long long mod_stride,
                                                          float eps, __nv_bfloat16* __restrict__ y, long long rows,
                                                          long long rows_per_b, int D) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int MAXP = 8;  // pieces of 8 values per lane: D <= 32 * 8 * 8 = 2048
  const int lane = threadIdx.x & 31;
  const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int np = D / 8;
  for (long long row = warp0; row < rows; row += nwarps) {
    const __nv_bfloat16* xr = x + row * D;
    float v[MAXP][8];
    float ss = 0.f;
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      const int piece = lane + 32 * p;
      if (piece < np) {
        ld8(xr + 8 * piece, v[p]);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(v[p][e], v[p][e], ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)D + eps);
    const long long b = row / rows_per_b;
    const float* sh = shift + b * mod_stride;
    const float* sc = scale + b * mod_stride;
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      const int piece = lane + 32 * p;
      if (piece < np) {
        float out[8];
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(sc + 8 * piece));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(sc + 8 * piece) + 1);
        const float4 h0 = __ldg(reinterpret_cast<const float4*>(sh + 8 * piece));
        const float4 h1 = __ldg(reinterpret_cast<const float4*>(sh + 8 * piece) + 1);
        const float scv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        const float shv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = fmaf(v[p][e] * inv, 1.f + scv[e], shv[e]);
        st8(y + row * D + 8 * piece, out);
      }
    }
  }
}

// x += gate[b] (*) y, 8 values per thread and step.
__global__ void __launch_bounds__(256) gated_add_kernel(__nv_bfloat16* __restrict__ x, const float* __restrict__ gate,
                                                        long long mod_stride, const __nv_bfloat16* __restrict__ y,
                                                        long long n8, long long per_b8, int D) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const long long b = i / per_b8;
    const int c0 = (int)((i * 8) % D);
    float xv[8], yv[8];
    ld8(x + 8 * i, xv);
    ld8(y + 8 * i, yv);
    const float4 ga = __ldg(reinterpret_cast<const float4*>(gate + b * mod_stride + c0));
    const float4 gb = __ldg(reinterpret_cast<const float4*>(gate + b * mod_stride + c0) + 1);
    const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) xv[e] = fmaf(gv[e], yv[e], xv[e]);
    st8(x + 8 * i, xv);
  }
}

// In place: SiLU (kind 0) or GELU, tanh form (kind 1), 8 values per thread and step.
__global__ void __launch_bounds__(256) act_kernel(__nv_bfloat16* __restrict__ x, long long n8, int kind) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    float v[8];
    ld8(x + 8 * i, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float a = v[e];
      if (kind == 0) {
        v[e] = a / (1.f + __expf(-a));
      } else {
        const float u = 0.7978845608028654f * (a + 0.044715f * a * a * a);
        v[e] = 0.5f * a * (1.f + tanhf(u));
      }
    }
    st8(x + 8 * i, v);
  }
}

int grid_for(long long work, int per_sm = 8) {
  const long long blocks = (work + 255) / 256;
  const long long cap = 148LL * per_sm;
  return (int)(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dig_status block_fail(dig_status s, const char* msg) {
  set_last_error(msg);
  return s;
}

dig_status launched(cudaError_t e) {
  if (e != cudaSuccess) return block_fail(DIG_ERR_CUDA, cudaGetErrorString(e));
  return DIG_OK;
}

}  // namespace
}  // namespace dig

using namespace dig;

extern "C" {

dig_status dig_block_rmsnorm_modulate(const void* x, const float* shift, const float* scale, long long mod_stride,
                                      float eps, void* y, int B, long long rows_per_batch, int D, void* stream) {
  if (B < 0 || rows_per_batch < 0 || D <= 0 || D % 8 != 0 || D > 2048)
    return block_fail(DIG_ERR_INVALID_ARGUMENT, "rmsnorm_modulate: D must be a multiple of 8 up to 2048");
  if (B == 0 || rows_per_batch == 0) return DIG_OK;
  if (!x || !shift || !scale || !y) return block_fail(DIG_ERR_INVALID_ARGUMENT, "rmsnorm_modulate: NULL tensor");
  if (!al16(x) || !al16(y) || !al16(shift) || !al16(scale) || mod_stride % 4 != 0)
    return block_fail(DIG_ERR_MISALIGNED, "rmsnorm_modulate: misaligned tensor or modulation row");
  const long long rows = (long long)B * rows_per_batch;
  return launched(launch_pdl(rmsnorm_mod_kernel, dim3(grid_for(rows * 32)), dim3(256), 0,
                             static_cast<cudaStream_t>(stream), static_cast<const __nv_bfloat16*>(x), shift, scale,
                             mod_stride, eps, static_cast<__nv_bfloat16*>(y), rows, rows_per_batch, D));
}

dig_status dig_block_gated_add(void* x, const float* gate, long long mod_stride, const void* y, int B,
                               long long rows_per_batch, int D, void* stream) {
  if (B < 0 || rows_per_batch < 0 || D <= 0 || D % 8 != 0)
    return block_fail(DIG_ERR_INVALID_ARGUMENT, "gated_add: D must be a positive multiple of 8");
  if (B == 0 || rows_per_batch == 0) return DIG_OK;
  if (!x || !gate || !y) return block_fail(DIG_ERR_INVALID_ARGUMENT, "gated_add: NULL tensor");
  if (!al16(x) || !al16(y) || !al16(gate) || mod_stride % 4 != 0)
    return block_fail(DIG_ERR_MISALIGNED, "gated_add: misaligned tensor or gate row");
  const long long n8 = (long long)B * rows_per_batch * D / 8;
  return launched(launch_pdl(gated_add_kernel, dim3(grid_for(n8)), dim3(256), 0, static_cast<cudaStream_t>(stream),
                             static_cast<__nv_bfloat16*>(x), gate, mod_stride, static_cast<const __nv_bfloat16*>(y),
                             n8, rows_per_batch * D / 8, D));
}

dig_status dig_block_activation(void* x, long long n, int kind, void* stream) {
  if (n < 0 || n % 8 != 0 || (kind != 0 && kind != 1))
    return block_fail(DIG_ERR_INVALID_ARGUMENT, "activation: n must be a multiple of 8, kind 0 or 1");
  if (n == 0) return DIG_OK;
  if (!x) return block_fail(DIG_ERR_INVALID_ARGUMENT, "activation: NULL tensor");
  if (!al16(x)) return block_fail(DIG_ERR_MISALIGNED, "activation: misaligned tensor");
  return launched(launch_pdl(act_kernel, dim3(grid_for(n / 8)), dim3(256), 0, static_cast<cudaStream_t>(stream),
                             static_cast<__nv_bfloat16*>(x), n / 8, kind));
}

}  // extern "C"
