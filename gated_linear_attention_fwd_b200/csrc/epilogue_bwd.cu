// epilogue_bwd.cu -- backward of the output gate and norm (DiG slides, "Gated
// Linear Attention Transformer (GLA) の導入", eq. (9)-(10)):
//
//   y_j = s_j * o_j * inv * gamma_j,   s_j = Swish(r_j) = r_j sigmoid(r_j),
//   inv = 1 / sqrt(mean_j(o_j^2) + eps)   (one row = one token of one head, d_v wide)
//
// For the upstream gradient dy, with a_j = dy_j s_j gamma_j:
//   d_o_j     = inv a_j - o_j inv^3 sum_m(a_m o_m) / d_v
//   d_r_j     = dy_j gamma_j o_j inv sigmoid(r_j) (1 + r_j (1 - sigmoid(r_j)))
//   d_gamma_j = sum over rows of dy_j s_j o_j inv
//
// HBM-bound: every row is read once (o, r, dy) and written once (d_o, d_r).
#include "dig_common.cuh"
#include "bwd_ops.h"
#include "gla_common.cuh"

namespace dig {

namespace {

// VEC consecutive values of a row: one 16-byte load (8 bf16 or 4 fp32 values).
template <typename T>
struct Row16;
template <>
struct Row16<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ __forceinline__ static void unpack(const uint4& u, float* o) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <>
struct Row16<float> {
  static constexpr int kVec = 4;
  __device__ __forceinline__ static void unpack(const uint4& u, float* o) {
    o[0] = __uint_as_float(u.x);
    o[1] = __uint_as_float(u.y);
    o[2] = __uint_as_float(u.z);
    o[3] = __uint_as_float(u.w);
  }
};

__device__ __forceinline__ void store4(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}
__device__ __forceinline__ void store4(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <int VEC, typename T>
__device__ __forceinline__ void store_vec(T* p, const float* v) {
  if constexpr (VEC == 8) st_global8(p, v);
  else store4(p, v);
}

// sigmoid by the hardware base-2 exponential; 0 for r below about -88, 1 above +17
__device__ __forceinline__ float sigmoid_fast(float r) { return __fdividef(1.f, 1.f + ex2(-r * kLog2e)); }

}  // namespace

// 16-byte asynchronous global -> shared copy, zero-filled when !valid (no bytes
// are read then; src must still be a valid address).
__device__ __forceinline__ void cp_async16_z(uint32_t saddr, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Row-group kernel.  A group of TPR threads owns one row (TPR = the power of two
// >= d_v / VEC): thread i holds columns VEC*i .. VEC*i+VEC-1 as one 16-byte vector
// (VEC = 8 bf16 or 4 fp32 values), so a warp's accesses cover 32 / TPR
// consecutive rows contiguously.  Each thread takes RPT rows per iteration and
// walks the rows with a grid-wide stride (the grid is the number of resident
// blocks).  The loads are a per-thread pipeline of NS stages in shared memory:
// every thread copies (cp.async, 16 bytes, zero-filled past the last row) exactly
// the vectors it will consume, NS - 1 iterations ahead, so no block barrier is
// needed and about NS * RPT * 48 bytes per thread stay in flight.  The two row
// sums (sum o^2 and sum a o) are reduced together with xor shuffles inside the
// group.  d_gamma: per-thread column partials, summed over the block's groups in
// shared memory, then one atomic add per column per block.
template <typename TIN, typename TOUT, int TPR, int RPT, int NS>
__global__ void __launch_bounds__(256) epilogue_bwd_kernel(const TIN* __restrict__ o, const TIN* __restrict__ r,
                                                           const float* __restrict__ gamma, float eps,
                                                           const TIN* __restrict__ dy, TOUT* __restrict__ d_o,
                                                           TOUT* __restrict__ d_r, float* __restrict__ d_gamma,
                                                           long long rows, int dv) {
  constexpr int VEC = Row16<TIN>::kVec;
  constexpr int GPB = 256 / TPR;  // row groups per block
  // pipe[stage][tensor: o, r, dy][u][thread], 16 bytes each
  extern __shared__ __align__(16) unsigned char epi_pipe[];
  __shared__ float sg[VEC * TPR];
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const int lane_g = threadIdx.x % TPR, grp = threadIdx.x / TPR;
  const int j0 = VEC * lane_g;
  const bool col_ok = j0 < dv;
  for (int i = threadIdx.x; i < VEC * TPR; i += blockDim.x) sg[i] = 0.f;
  float gm[VEC], acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    gm[e] = (gamma && col_ok) ? __ldg(gamma + j0 + e) : 1.f;
    acc[e] = 0.f;
  }
  const float inv_dv = 1.f / (float)dv;
  const long long stride = (long long)gridDim.x * GPB;
  const long long first = (long long)blockIdx.x * GPB;
  const long long niter = first < rows ? (rows - first + stride * RPT - 1) / (stride * RPT) : 0;
  const uint32_t slot0 = smem_u32(epi_pipe) + 16u * threadIdx.x;
  auto slot = [&](int st, int tn, int u) -> uint32_t { return slot0 + 16u * 256u * (uint32_t)((st * 3 + tn) * RPT + u); };
  auto issue = [&](long long k) {
    if (k >= niter) return;
    const int st = (int)(k % NS);
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      const long long row = first + k * stride * RPT + grp + u * stride;
      const bool ok = col_ok && row < rows;
      const size_t off = ok ? (size_t)row * dv + j0 : 0;
      cp_async16_z(slot(st, 0, u), o + off, ok);
      cp_async16_z(slot(st, 1, u), r + off, ok);
      cp_async16_z(slot(st, 2, u), dy + off, ok);
    }
  };
#pragma unroll
  for (int k = 0; k < NS - 1; ++k) {
    issue(k);
    cp_async_commit();
  }
  for (long long k = 0; k < niter; ++k) {
    issue(k + NS - 1);
    cp_async_commit();
    cp_async_wait_group<NS - 1>();  // this thread's copies of iteration k have landed
    const int st = (int)(k % NS);
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      float ov[VEC], rv[VEC], gv[VEC], sig[VEC], a[VEC];
      uint4 raw[3];
#pragma unroll
      for (int tn = 0; tn < 3; ++tn)
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(raw[tn].x), "=r"(raw[tn].y), "=r"(raw[tn].z), "=r"(raw[tn].w)
                     : "r"(slot(st, tn, u)));
      Row16<TIN>::unpack(raw[0], ov);
      Row16<TIN>::unpack(raw[1], rv);
      Row16<TIN>::unpack(raw[2], gv);
      float s1 = 0.f, s2 = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        sig[e] = sigmoid_fast(rv[e]);
        a[e] = gv[e] * rv[e] * sig[e] * gm[e];
        s1 = fmaf(ov[e], ov[e], s1);
        s2 = fmaf(a[e], ov[e], s2);
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) {
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
        s2 += __shfl_xor_sync(0xffffffffu, s2, off);
      }
      const long long row = first + k * stride * RPT + grp + u * stride;
      if (!col_ok || row >= rows) continue;
      const float inv = rsqrtf(s1 * inv_dv + eps);
      const float c = inv * inv * inv * s2 * inv_dv;
      float vo[VEC], vr[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float n = ov[e] * inv;
        vo[e] = inv * a[e] - ov[e] * c;
        vr[e] = gv[e] * gm[e] * n * sig[e] * (1.f + rv[e] * (1.f - sig[e]));
        acc[e] = fmaf(gv[e] * rv[e] * sig[e], n, acc[e]);
      }
      const size_t off = (size_t)row * dv + j0;
      store_vec<VEC>(d_o + off, vo);
      store_vec<VEC>(d_r + off, vr);
    }
  }
  cp_async_wait_group<0>();
  if (!d_gamma) return;
  __syncthreads();  // sg zeroed
  if (col_ok)
#pragma unroll
    for (int e = 0; e < VEC; ++e) atomicAdd(&sg[j0 + e], acc[e]);
  __syncthreads();
  for (int j = threadIdx.x; j < dv; j += blockDim.x) atomicAdd(d_gamma + j, sg[j]);
}

// Any d_v: one warp per row, two passes over the row (sums, then outputs; the
// second pass reads the row again from L1/L2); d_gamma partials in shared memory.
template <typename TIN, typename TOUT>
__global__ void __launch_bounds__(256) epilogue_bwd_generic_kernel(const TIN* __restrict__ o,
                                                                   const TIN* __restrict__ r,
                                                                   const float* __restrict__ gamma, float eps,
                                                                   const TIN* __restrict__ dy, TOUT* __restrict__ d_o,
                                                                   TOUT* __restrict__ d_r,
                                                                   float* __restrict__ d_gamma, long long rows,
                                                                   int dv) {
  extern __shared__ float sg_dyn[];
  griddep_wait();  // the kernels before this one have completed
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int j = threadIdx.x; j < dv; j += blockDim.x) sg_dyn[j] = 0.f;
  __syncthreads();
  const float inv_dv = 1.f / (float)dv;
  for (long long row = (long long)blockIdx.x * 8 + warp; row < rows; row += (long long)gridDim.x * 8) {
    const size_t base = (size_t)row * dv;
    float s1 = 0.f, s2 = 0.f;
    for (int j = lane; j < dv; j += 32) {
      const float ov = (float)o[base + j], rv = (float)r[base + j], gv = (float)dy[base + j];
      const float g = gamma ? __ldg(gamma + j) : 1.f;
      s1 = fmaf(ov, ov, s1);
      s2 = fmaf(gv * rv * sigmoid_fast(rv) * g, ov, s2);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      s2 += __shfl_xor_sync(0xffffffffu, s2, off);
    }
    const float inv = rsqrtf(s1 * inv_dv + eps);
    const float c = inv * inv * inv * s2 * inv_dv;
    for (int j = lane; j < dv; j += 32) {
      const float ov = (float)o[base + j], rv = (float)r[base + j], gv = (float)dy[base + j];
      const float g = gamma ? __ldg(gamma + j) : 1.f;
      const float sig = sigmoid_fast(rv), n = ov * inv;
      d_o[base + j] = static_cast<TOUT>(inv * gv * rv * sig * g - ov * c);
      d_r[base + j] = static_cast<TOUT>(gv * g * n * sig * (1.f + rv * (1.f - sig)));
      if (d_gamma) atomicAdd(&sg_dyn[j], gv * rv * sig * n);
    }
  }
  if (!d_gamma) return;
  __syncthreads();
  for (int j = threadIdx.x; j < dv; j += blockDim.x) atomicAdd(d_gamma + j, sg_dyn[j]);
}

namespace {

// Rows per thread per iteration and pipeline stages: 2 x 4 stages x 3 tensors x
// 16 bytes x 256 threads = 96 KB of shared memory per block, two blocks per SM.
constexpr int kEpiRowsPerThread = 2, kEpiStages = 4;

template <typename TIN, typename TOUT, int TPR>
cudaError_t launch_rows(const void* o, const void* r, const float* gamma, float eps, const void* dy, void* d_o,
                        void* d_r, float* d_gamma, long long rows, int dv, int sms, cudaStream_t s) {
  constexpr int GPB = 256 / TPR, RPT = kEpiRowsPerThread, NS = kEpiStages;
  constexpr size_t smem = (size_t)NS * 3 * RPT * 256 * 16;
  auto kern = epilogue_bwd_kernel<TIN, TOUT, TPR, RPT, NS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess || per_sm < 1) per_sm = 1;
  const long long need = (rows + (long long)GPB * RPT - 1) / ((long long)GPB * RPT);
  const int grid = (int)(need < (long long)sms * per_sm ? need : (long long)sms * per_sm);
  return launch_pdl(kern, dim3(grid), dim3(256), smem, s, reinterpret_cast<const TIN*>(o),
                    reinterpret_cast<const TIN*>(r), gamma, eps, reinterpret_cast<const TIN*>(dy),
                    reinterpret_cast<TOUT*>(d_o), reinterpret_cast<TOUT*>(d_r), d_gamma, rows, dv);
}

template <typename TIN, typename TOUT>
cudaError_t launch_epi_typed(const void* o, const void* r, const float* gamma, float eps, const void* dy, void* d_o,
                             void* d_r, float* d_gamma, long long rows, int dv, cudaStream_t s) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int VEC = Row16<TIN>::kVec;
  if (dv % VEC == 0 && dv <= 32 * VEC) {
    const int groups = dv / VEC;
    if (groups <= 4) return launch_rows<TIN, TOUT, 4>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, sms, s);
    if (groups <= 8) return launch_rows<TIN, TOUT, 8>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, sms, s);
    if (groups <= 16) return launch_rows<TIN, TOUT, 16>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, sms, s);
    return launch_rows<TIN, TOUT, 32>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, sms, s);
  }
  const long long need = (rows + 7) / 8;
  const int grid = (int)(need < (long long)sms * 8 ? need : (long long)sms * 8);
  return launch_pdl(epilogue_bwd_generic_kernel<TIN, TOUT>, dim3(grid), dim3(256), (size_t)dv * 4, s,
                    reinterpret_cast<const TIN*>(o), reinterpret_cast<const TIN*>(r), gamma, eps,
                    reinterpret_cast<const TIN*>(dy), reinterpret_cast<TOUT*>(d_o), reinterpret_cast<TOUT*>(d_r),
                    d_gamma, rows, dv);
}

}  // namespace

cudaError_t launch_epilogue_bwd(const void* o, const void* r, const float* gamma, float eps, const void* dy,
                                void* d_o, void* d_r, float* d_gamma, long long rows, int dv, int tin, int tout,
                                cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (d_gamma) {
    const cudaError_t e = cudaMemsetAsync(d_gamma, 0, (size_t)dv * sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  if (rows == 0) return cudaSuccess;
  if (tin == DIG_BF16) {
    if (tout == DIG_BF16) return launch_epi_typed<bf, bf>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, s);
    return launch_epi_typed<bf, float>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, s);
  }
  if (tout == DIG_BF16) return launch_epi_typed<float, bf>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, s);
  return launch_epi_typed<float, float>(o, r, gamma, eps, dy, d_o, d_r, d_gamma, rows, dv, s);
}

}  // namespace dig
