// sq_tmap.h -- host-side TMA tensor-map construction for int8 row-major
// matrices (K contiguous), 128-byte swizzle, zero fill out of bounds.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "sq_internal.h"

namespace sq {

// rows x K int8 matrix at `base` (row stride K bytes); boxes of
// box_k bytes along K x box_rows rows, stored with the swizzle whose span is
// box_k bytes (128 -> 128-byte swizzle, 64 -> 64-byte swizzle).
inline bool make_tmap_i8(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows,
                         uint32_t box_k, uint32_t box_rows) {
  const CUtensorMapSwizzle swz = box_k == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!encode) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K};
  cuuint32_t box[2] = {box_k, box_rows};
  cuuint32_t elem[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                      box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// rows x cols fp16 matrix (row stride cols * 2 bytes, a multiple of 16), boxes
// of 32 x 32 elements stored with the 64-byte swizzle (the shared-memory
// image is 32 rows of 64 bytes, 16-byte chunk c of row r at chunk
// c ^ ((r >> 1) & 3)).
inline bool make_tmap_f16_out(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows) {
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!encode) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t elem[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                      box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sq

namespace sq {

// batch x rows x K int8 tensor (K contiguous, batch items rows * K apart);
// boxes of box_k x box_rows x 1, 128-byte swizzle (box_k = 128).
inline bool make_tmap_i8_3d(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint64_t batch,
                            uint32_t box_k, uint32_t box_rows) {
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!encode) return false;
  cuuint64_t dims[3] = {K, rows, batch};
  cuuint64_t strides[2] = {K, K * rows};
  cuuint32_t box[3] = {box_k, box_rows, 1};
  cuuint32_t elem[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                      elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// batch x rows x cols fp16 output (row stride cols * 2 bytes, a multiple of
// 16), 32 x 32 x 1 boxes with the 64-byte swizzle of make_tmap_f16_out.
inline bool make_tmap_f16_out_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                                 uint64_t batch) {
  auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
  if (!encode) return false;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t elem[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                      elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sq
