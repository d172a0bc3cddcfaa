// tma_tiles.cuh -- pieces shared by the kernels that move whole token tiles by
// TMA: where a unit's tile sits in the token tensors, and shared-memory access
// helpers for the swizzled tiles.
#pragma once
#include <cuda_fp16.h>

#include "gla_chunk.cuh"
#include "tma.cuh"
#include "tmap.h"

namespace dig {

// Tile placement of a unit: the chunk's C tokens as a box of consecutive grid
// tokens (row orders) or as C / 16 column segments (column orders).  `rev`: the
// tile's rows run against the scan order (tile row i is scan position C-1-i).
struct TileUnit {
  int b, h, n, bz, hz;
  bool rev, col;
  int y;   // row orders: first grid token of the box, as a row of the [B * L] view
  int q0;  // column orders: first column-order position of the tile
  __device__ TileUnit(const GlaArgs& a, int u, int C) {
    const int bh = u / a.nchunks;
    n = u - bh * a.nchunks;
    b = bh / a.H;
    h = bh - b * a.H;
    bz = b * a.gate_heads + (a.gate_heads == 1 ? 0 : h);
    hz = a.gate_heads == 1 ? 0 : h;
    rev = (a.mode & 1) != 0;
    col = (a.mode & 2) != 0;
    const int first = rev ? a.L - (n + 1) * C : n * C;
    y = b * a.L + first;
    q0 = first;
  }
  // column segment j: grid row and column of its first token
  __device__ void seg(const GlaArgs& a, int j, int& row, int& cl) const {
    const int p = q0 + 16 * j;
    cl = p / a.Hg;
    row = p - cl * a.Hg;
  }
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float h_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu))); }
__device__ __forceinline__ float h_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// A unit's C-row tile of one head slice (x: the slice's first element within a
// token row; rb: bytes of one tile row) as one box (row orders) or C / 16
// column segments (column orders).
template <int C>
__device__ __forceinline__ void tile_load(uint32_t dst, const CUtensorMap& m, int x, const TileUnit& T,
                                          const GlaArgs& a, int rb, uint64_t* bar) {
  if (!T.col) {
    tma_load_2d(dst, m, x, T.y, bar);
  } else {
    for (int j = 0; j < C / 16; ++j) {
      int row, cl;
      T.seg(a, j, row, cl);
      tma_load_4d(dst + j * 16 * rb, m, x, row, cl, T.b, bar);
    }
  }
}
template <int C>
__device__ __forceinline__ void tile_store(const CUtensorMap& m, int x, const TileUnit& T, const GlaArgs& a,
                                           uint32_t src, int rb) {
  if (!T.col) {
    tma_store_2d(m, x, T.y, src);
  } else {
    for (int j = 0; j < C / 16; ++j) {
      int row, cl;
      T.seg(a, j, row, cl);
      tma_store_4d(m, x, row, cl, T.b, src + j * 16 * rb);
    }
  }
}

// Host: the tile map of a token tensor with rows of `row_elems` elements, for
// the scan order of `a` (boxes of C consecutive tokens, or 16-row column segments).
inline bool encode_tile_map(CUtensorMap* m, const void* p, CUtensorMapDataType dt, int esize, int row_elems,
                            uint32_t box_elems, int rb, const GlaArgs& a, int C) {
  if (a.mode & 2) return tmap_cols(m, p, dt, esize, row_elems, a.Hg, a.Wg, a.B, box_elems, 16, rb);
  return tmap_rows(m, p, dt, esize, row_elems, (uint64_t)a.B * a.L, box_elems, C, rb);
}

}  // namespace dig
