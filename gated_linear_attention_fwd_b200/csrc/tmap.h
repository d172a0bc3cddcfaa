// tmap.h -- TMA tensor maps over the library's token tensors (host side).
//
// Every token tensor is [B, L, H', D] in grid row-major token order with rows of
// `row_elems` = H' * D elements.  Two views are encoded:
//   rows: 2-D (row_elems, B * L); a box is `box_rows` consecutive tokens of one
//         head slice (x = head * D, y = b * L + first token) -- the row scan orders;
//   cols: 4-D (row_elems, grid row, grid column, image); a box is `box_rows`
//         consecutive grid rows of one grid column -- the column scan orders.
// Both use the 64- or 128-byte swizzle (`rb`, the bytes of one box row).
#pragma once
#include <cuda.h>

#include <cstdint>

namespace dig {

bool tmap_available();
bool tmap_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t row_elems,
               uint64_t rows, uint32_t box_elems, uint32_t box_rows, int rb);
bool tmap_cols(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t row_elems, int Hg, int Wg,
               int B, uint32_t box_elems, uint32_t box_rows, int rb);

}  // namespace dig
