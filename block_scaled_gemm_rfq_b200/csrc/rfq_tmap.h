// rfq_tmap.h -- TMA tensor maps over the packed MXFP4 operands, shared by the
// GEMM and the fused linear kernel (host code).
#pragma once

#include <cuda.h>

#include <cstdint>

namespace rfq {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D map over code rows of row_bytes bytes ([rows][row_bytes]); box = 128 bytes x
// box_rows rows, 128-byte swizzle (the layout operand_desc() describes), zero fill
// outside.
inline bool encode_code_rows_map(EncodeTiledFn encode, CUtensorMap* map, const void* codes, int64_t rows,
                                 int64_t row_bytes, uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t elem_strides[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, elem_strides,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same over packed FP4 codes [rows][K/2].
inline bool encode_codes_map(EncodeTiledFn encode, CUtensorMap* map, const void* codes, int64_t rows, int64_t K,
                             uint32_t box_rows) {
  return encode_code_rows_map(encode, map, codes, rows, K / 2, box_rows);
}

// 4-D map over a scale array in the MMA layout: [row tiles][k atoms][2][256 B]
// (a 512-byte atom = 128 rows x 4 blocks = 128 K).  The box takes `box_katoms`
// consecutive k-atoms (2: a 256-K FP4 stage; 1: a 128-K FP8 stage) of `box_tiles`
// consecutive row tiles; atoms past the end in either direction read as zeros.
inline bool encode_scales_map(EncodeTiledFn encode, CUtensorMap* map, const void* scales, int64_t rows,
                              int64_t K, uint32_t box_tiles, uint32_t box_katoms = 2) {
  const int64_t row_tiles = (rows + 127) / 128;
  const int64_t k_atoms = (K / 32 + 3) / 4;
  cuuint64_t dims[4] = {256, 2, static_cast<cuuint64_t>(k_atoms), static_cast<cuuint64_t>(row_tiles)};
  cuuint64_t strides[3] = {256, 512, static_cast<cuuint64_t>(k_atoms * 512)};
  cuuint32_t box[4] = {256, 2, box_katoms, box_tiles};
  cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(scales), dims, strides, box, elem_strides,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace rfq
