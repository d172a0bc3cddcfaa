// gla_common.cuh -- device helpers shared by the GLA forward and backward
// kernels: compile-time sizes, split-term bf16 operand stores, prefetch vectors,
// the base-2 gate, and the tensor-core issue loop.
#pragma once
#include <cstring>
#include <type_traits>

#include "dig_common.cuh"
#include "sm100.cuh"

namespace dig {

__host__ __device__ constexpr int cround(int x, int m) { return (x + m - 1) / m * m; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int pow2ceil(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

// Store one operand value as NT bf16 terms (term i in copy i).
template <int NT>
__device__ __forceinline__ void st_op(uint8_t* base, int copy_bytes, uint32_t off, float x) {
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const __nv_bfloat16 hb = __float2bfloat16_rn(x);
    *reinterpret_cast<__nv_bfloat16*>(base + i * copy_bytes + off) = hb;
    x -= __bfloat162float(hb);
  }
}
// Four consecutive K values of one row (8 bytes per term, same core-matrix row).
template <int NT>
__device__ __forceinline__ void st_op4(uint8_t* base, int copy_bytes, uint32_t off, float x0, float x1, float x2,
                                       float x3) {
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x0, x1);
    const __nv_bfloat162 b = __floats2bfloat162_rn(x2, x3);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&a);
    u.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(base + i * copy_bytes + off) = u;
    x0 -= __low2float(a);
    x1 -= __high2float(a);
    x2 -= __low2float(b);
    x3 -= __high2float(b);
  }
}

// Shared-space stores of split bf16 terms: `saddr` is a shared-memory address
// (cvta), term i goes to saddr + i * copy_bytes.
template <int NT>
__device__ __forceinline__ void sts_op4(uint32_t saddr, uint32_t copy_bytes, const float* x) {
  float r[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(r[0], r[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(r[2], r[3]);
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(saddr + i * copy_bytes),
                 "r"(*reinterpret_cast<const uint32_t*>(&a)), "r"(*reinterpret_cast<const uint32_t*>(&b))
                 : "memory");
    r[0] -= __low2float(a);
    r[1] -= __high2float(a);
    r[2] -= __low2float(b);
    r[3] -= __high2float(b);
  }
}
template <int NT>
__device__ __forceinline__ void sts_op8(uint32_t saddr, uint32_t copy_bytes, const float* x) {
  float r[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) r[j] = x[j];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) h[j] = __floats2bfloat162_rn(r[2 * j], r[2 * j + 1]);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr + i * copy_bytes),
                 "r"(*reinterpret_cast<const uint32_t*>(&h[0])), "r"(*reinterpret_cast<const uint32_t*>(&h[1])),
                 "r"(*reinterpret_cast<const uint32_t*>(&h[2])), "r"(*reinterpret_cast<const uint32_t*>(&h[3]))
                 : "memory");
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      r[2 * j] -= __low2float(h[j]);
      r[2 * j + 1] -= __high2float(h[j]);
    }
  }
}
// Writes channels C0 .. C0+N-1 (C0, N multiples of 4) of one operand row in the
// K-major layout: 16-byte stores where a core-matrix row (8 channels) is
// covered, 8-byte stores for half rows.  `row` is the shared address of
// channel 0 of the row.
template <int NT, int C0, int N>
struct RowWriter {
  __device__ __forceinline__ static void run(uint32_t row, uint32_t copy_bytes, const float* x) {
    if constexpr (N <= 0) {
      return;
    } else if constexpr (C0 % 8 == 0 && N >= 8) {
      sts_op8<NT>(row + (C0 / 8) * 128, copy_bytes, x);
      RowWriter<NT, C0 + 8, N - 8>::run(row, copy_bytes, x + 8);
    } else {
      sts_op4<NT>(row + (C0 / 8) * 128 + (C0 % 8) * 2, copy_bytes, x);
      RowWriter<NT, C0 + 4, N - 4>::run(row, copy_bytes, x + 4);
    }
  }
};
// Shared address of row t's channel 0 in a K-major buffer with row stride sbo.
__device__ __forceinline__ uint32_t row_addr(uint32_t buf, int t, int sbo) {
  return buf + (uint32_t)(t >> 3) * sbo + (uint32_t)(t & 7) * 16u;
}

__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

// Coalesced work split of a [rows][NG] grid of row pieces over a CTA: piece i
// is (row, group) with runs of 8 consecutive rows per group, so a warp touches
// 8 rows x 4 groups (few cache lines per load) and every 8-lane phase of a
// 16-byte shared-memory store covers 8 consecutive K-major rows (no bank
// conflicts).
template <int NG>
__device__ __forceinline__ void piece_of(int i, int& row, int& g) {
  const int rest = i >> 3;
  g = rest % NG;
  row = (rest / NG) * 8 + (i & 7);
}

// PS consecutive elements of one row as raw 32-bit words (vector loads).
template <typename T, int PS>
struct Piece {
  static constexpr int NW = PS * (int)sizeof(T) / 4;
  static_assert(NW == 2 || NW % 4 == 0, "8-byte or whole 16-byte pieces");
  uint32_t w[NW];
  __device__ __forceinline__ void load(const T* p, bool valid) {
    if constexpr (NW == 2) {
      const uint2 u = valid ? __ldg(reinterpret_cast<const uint2*>(p)) : make_uint2(0u, 0u);
      w[0] = u.x;
      w[1] = u.y;
    } else {
#pragma unroll
      for (int i = 0; i < NW; i += 4) {
        const uint4 u = valid ? __ldg(reinterpret_cast<const uint4*>(p) + i / 4) : make_uint4(0u, 0u, 0u, 0u);
        w[i] = u.x;
        w[i + 1] = u.y;
        w[i + 2] = u.z;
        w[i + 3] = u.w;
      }
    }
  }
  // L2-only load of data written earlier in the same stream by another kernel
  __device__ __forceinline__ void load_cg(const T* p, bool valid) {
#pragma unroll
    for (int i = 0; i < NW; i += 4) {
      const uint4 u = valid ? __ldcg(reinterpret_cast<const uint4*>(p) + i / 4) : make_uint4(0u, 0u, 0u, 0u);
      w[i] = u.x;
      w[i + 1] = u.y;
      w[i + 2] = u.z;
      w[i + 3] = u.w;
    }
  }
  __device__ __forceinline__ void unpack(float* o) const {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < NW; ++i) o[i] = __uint_as_float(w[i]);
    }
  }
};

// Stores PS values (PS = 4 or 8) at channel c0 (c0 % PS == 0) of row `row` of a
// K-major operand buffer, as NT bf16 terms.
template <int NT, int PS>
__device__ __forceinline__ void st_piece(uint32_t buf, int row, int sbo, int c0, uint32_t copy_bytes,
                                         const float* x) {
  const uint32_t a = row_addr(buf, row, sbo) + (uint32_t)(c0 >> 3) * 128u + (uint32_t)(c0 & 7) * 2u;
  if constexpr (PS == 8) sts_op8<NT>(a, copy_bytes, x);
  else sts_op4<NT>(a, copy_bytes, x);
}

// Stores 8 values to global memory as bf16 (one 16-byte store) or fp32 (two).
__device__ __forceinline__ void st_global8(__nv_bfloat16* p, const float* v) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]);
  u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]);
  u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void st_global8(float* p, const float* v) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Raw 4-element vectors as fetched from global memory (prefetched in registers).
template <typename T>
struct Raw4;
template <>
struct Raw4<__nv_bfloat16> {
  using type = uint2;
};
template <>
struct Raw4<float> {
  using type = float4;
};
__device__ __forceinline__ void unpack4(const uint2& u, float* o) {
  o[0] = __uint_as_float(u.x << 16);
  o[1] = __uint_as_float(u.x & 0xFFFF0000u);
  o[2] = __uint_as_float(u.y << 16);
  o[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ void unpack4(const float4& u, float* o) {
  o[0] = u.x;
  o[1] = u.y;
  o[2] = u.z;
  o[3] = u.w;
}
template <typename R>
__device__ __forceinline__ R zero4() {
  R r;
  memset(&r, 0, sizeof(R));
  return r;
}

constexpr float kLog2e = 1.4426950408889634f;
// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz.f32:
// a few ulp; results below 2^-126 flush to 0).  The gate factors stay within
// 2^+-115 (checked), so only the contributions of tokens decayed by more than
// 2^-126 are affected, and those are negligible.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Base-2 log decay of one gate logit: inv_tau * log2(sigmoid(z)), evaluated as
// inv_tau * (min(z, 0) * log2(e) - log2(1 + 2^(-|z| log2(e)))).  The logarithm's
// argument lies in (1, 2], where the fast __log2f is accurate to about 2^-22.
__device__ __forceinline__ float log2_decay(float z, float inv_tau) {
  return inv_tau * (fminf(z, 0.f) * kLog2e - __log2f(1.f + ex2(-fabsf(z) * kLog2e)));
}

// Issues D (+)= A * B for operands stored as NA / NB bf16 terms: every term
// pair (i, j) with i + j below max(NA, NB), KSTEPS K-steps each.  Descriptors
// are formed once; later K-steps and terms only add to the start-address field
// (shared-memory addresses stay below 2^18, so the 14-bit field never carries).
template <int NA, int NB, int KSTEPS>
__device__ __forceinline__ void mma_issue(uint32_t dtm, uint64_t a0, uint32_t a_term, uint32_t a_kstep, uint64_t b0,
                                          uint32_t b_term, uint32_t b_kstep, uint32_t idesc, bool accumulate) {
  constexpr int ORD = NA > NB ? NA : NB;
  bool first = !accumulate;
#pragma unroll
  for (int i = 0; i < NA; ++i) {
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (i + j >= ORD) continue;
#pragma unroll
      for (int s = 0; s < KSTEPS; ++s) {
        mma_bf16(dtm, a0 + (uint64_t)((i * a_term + s * a_kstep) >> 4), b0 + (uint64_t)((j * b_term + s * b_kstep) >> 4),
                 idesc, first ? 0u : 1u);
        first = false;
      }
    }
  }
}


// The per-thread program.  Threads 0-127 own channel half 0, threads 128-255
// half 1 (compile-time H); both halves run the same barrier sequence.

}  // namespace dig
