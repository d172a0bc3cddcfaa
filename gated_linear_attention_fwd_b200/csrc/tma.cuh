// tma.cuh -- tensor-memory-accelerator (TMA) tile copies and the swizzled shared-
// memory layouts they produce, for the kernels that move whole tiles
// asynchronously instead of by per-thread loads and stores.
//
// A tile is `rows` token rows of one head slice (RB bytes per row: 64 or 128).
// TMA writes it to shared memory with the 64-byte or 128-byte swizzle: row i
// occupies RB contiguous bytes at i * RB, and its 16-byte chunk c is stored at
// chunk position c ^ f(i), with f(i) = i % 8 for RB = 128 and (i / 2) % 4 for
// RB = 64 (the swizzle acts on the shared-memory address bits, so tiles start
// at 1024-byte boundaries).  The same bytes are a valid tensor-core operand in
// the swizzled K-major layout (8-row groups RB * 8 bytes apart, a K-step of 16
// 2-byte values = +32 bytes) and, read with rows as the contracted dimension, in
// the swizzled MN-major layout (a K-step of 16 rows = +16 * RB bytes).
#pragma once
#include <cuda.h>
#include <cstdint>

#include "sm100.cuh"

namespace dig {

// Byte offset of 16-byte chunk c of row i in a swizzled tile of RB-byte rows.
template <int RB>
__host__ __device__ __forceinline__ uint32_t swz_off(uint32_t i, uint32_t c) {
  static_assert(RB == 64 || RB == 128, "64- or 128-byte rows");
  if constexpr (RB == 128) return i * 128u + ((c ^ (i & 7u)) << 4);
  else return i * 64u + ((c ^ ((i >> 1) & 3u)) << 4);
}

// Shared-memory matrix descriptor of a swizzled operand: SBO = 8 rows, layout 2
// (128-byte swizzle) or 4 (64-byte swizzle).  The leading-byte offset is not
// used by these layouts (one swizzle atom spans the whole row); it is set equal
// to SBO.
template <int RB>
__device__ __forceinline__ uint64_t sdesc_sw(uint32_t saddr) {
  constexpr uint32_t sbo = 8u * RB;
  constexpr uint64_t layout = RB == 128 ? 2u : 4u;
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= layout << 61;
  return d;
}

// Instruction descriptor: kind::f16 with fp16 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn = false, bool b_mn = false) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Adds `bytes` to the transaction count of the barrier's current phase, without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t tmap_addr(const CUtensorMap& m) { return reinterpret_cast<uint64_t>(&m); }

// ---- loads (global -> this CTA's shared memory, completing as transactions on `bar`; no multicast)
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap& m, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(tmap_addr(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap& m, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(dst),
      "l"(tmap_addr(m)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}
// ---- stores and fp32 add-reductions (shared -> global), tracked by bulk groups
__device__ __forceinline__ void tma_store_2d(const CUtensorMap& m, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap_addr(m)), "r"(x),
               "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap& m, int x, int y, int z, int w, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(tmap_addr(m)),
               "r"(x), "r"(y), "r"(z), "r"(w), "r"(src)
               : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap& m, int x, int y, uint32_t src) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   tmap_addr(m)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap& m, int x, int y, int z, int w, uint32_t src) {
  asm volatile("cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
                   tmap_addr(m)),
               "r"(x), "r"(y), "r"(z), "r"(w), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Every committed bulk group has finished reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Two fp32 -> packed fp16x2 (round to nearest; out-of-range values become +-inf).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Running maximum of |x| over packed fp16x2 values (inf and NaN propagate as large).
__device__ __forceinline__ uint32_t absmax_f16x2(uint32_t acc, uint32_t x) {
  uint32_t r;
  const uint32_t ax = x & 0x7FFF7FFFu;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(ax));
  return r;
}
// True when a running |x| maximum (absmax_f16x2) reached 2^15 or more, or held inf / NaN.
__device__ __forceinline__ bool f16x2_too_large(uint32_t acc) {
  return ((acc & 0xFFFFu) >= 0x7800u) || ((acc >> 16) >= 0x7800u);
}

}  // namespace dig
