// tmap.cu -- host-side encoding of the TMA tensor maps (cuTensorMapEncodeTiled,
// reached through the runtime's driver entry point, so the library links no
// driver library of its own).
#include <cuda_runtime.h>

#include <mutex>

#include "tmap.h"

namespace dig {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUtensorMapSwizzle swizzle_of(int rb) { return rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B; }

}  // namespace

bool tmap_available() { return encode_fn() != nullptr; }

bool tmap_rows(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t row_elems,
               uint64_t rows, uint32_t box_elems, uint32_t box_rows, int rb) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {row_elems, rows};
  const cuuint64_t strides[1] = {row_elems * (uint64_t)esize};
  const cuuint32_t box[2] = {box_elems, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(rb),
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tmap_cols(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t row_elems, int Hg, int Wg,
               int B, uint32_t box_elems, uint32_t box_rows, int rb) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t pitch = row_elems * (uint64_t)esize;  // bytes of one grid token
  const cuuint64_t dims[4] = {row_elems, (cuuint64_t)Hg, (cuuint64_t)Wg, (cuuint64_t)B};
  const cuuint64_t strides[3] = {pitch * (uint64_t)Wg, pitch, pitch * (uint64_t)Wg * (uint64_t)Hg};
  const cuuint32_t box[4] = {box_elems, box_rows, 1, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(rb),
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dig
