// Host-side construction of TMA tensor maps (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so libda.so does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace da {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_tiled();

// A [depth][rows][inner] bf16 tensor (inner contiguous) read in boxes of box_rows x box_inner
// elements, with the 128-byte swizzle (box_inner = 64) or none; out-of-range rows read as zero.
inline bool make_tmap_bf16_3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t depth,
                              uint32_t box_inner, uint32_t box_rows, bool swizzle128 = true) {
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {inner * 2, inner * 2 * rows};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 tensor of `depth` tiles, each `rows` x `inner` (inner contiguous, rows `inner`*2 bytes
// apart), tiles `tile_stride` bytes apart; boxes of box_rows x 64 elements, 128-byte swizzle.
inline bool make_tmap_bf16_tiles(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t depth,
                                 uint64_t tile_stride, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {inner * 2, tile_stride};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace da
