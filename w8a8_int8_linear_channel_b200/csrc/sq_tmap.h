// sq_tmap.h -- host-side TMA tensor-map construction for int8 row-major
// matrices (K contiguous), 128-byte swizzle, zero fill out of bounds.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "sq_internal.h"

namespace sq {

// rows x K int8 matrix at `base` (row stride K bytes); boxes of
// box_k (bytes along K, <= 128 for the 128-byte swizzle) x box_rows rows.
inline bool make_tmap_i8(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows,
                         uint32_t box_k, uint32_t box_rows) {
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!encode) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K};
  cuuint32_t box[2] = {box_k, box_rows};
  cuuint32_t elem[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                      box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sq
