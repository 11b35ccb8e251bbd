// Host helper: 2D TMA tensor maps (bf16, 128-byte swizzle) through the driver entry point
// cuTensorMapEncodeTiled, looked up once via the runtime (no libcuda link dependency).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

namespace rdl {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return (EncodeTiledFn)p;
  }();
  return fn;
}

// Row-major bf16 matrix [rows x cols] at `base` (16-byte aligned, cols*2 a multiple of 16);
// boxes of box_cols x box_rows land in shared memory with the 128-byte swizzle
// (box_cols * 2 must be 128).  Rows past the end read as zeros.
inline bool make_tmap_bf16(CUtensorMap* map, const void* base, unsigned long long rows, unsigned cols,
                           unsigned box_cols, unsigned box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K or V of one KV head as [rows x 128] bf16 (row stride 256 B), viewed as (64 columns,
// rows, 2 halves) so that one box of box_rows rows x 2 halves lands as two 128-byte-swizzled
// tiles of box_rows x 128 B (columns 0-63, then 64-127).
inline bool make_tmap_kv_halves(CUtensorMap* map, const void* base, unsigned long long rows,
                                unsigned box_rows = 64) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, rows, 2};
  cuuint64_t strides[2] = {256, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Any bf16 view with a 64-element (128-byte) innermost box dimension, 128-byte swizzle:
// dims[0] = 64 columns, dims/strides (bytes) of the outer dimensions as given.  Outside the
// tensor reads as zeros.
inline bool make_tmap_bf16_nd(CUtensorMap* map, const void* base, unsigned nd, const cuuint64_t* dims,
                              const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, nd, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Queries q [tokens, Hq, 128] bf16 viewed as (64 columns, Hq heads, 2 halves, tokens): one box
// of 8 heads x 2 halves x R consecutive tokens lands token-major, 2 KB per token (half 0 of
// its 8 head rows, then half 1), each 1 KB a 128-byte-swizzled tile.  Heads past Hq read as 0.
inline bool make_tmap_q_run(CUtensorMap* map, const void* base, unsigned long long tokens, unsigned Hq,
                            unsigned run) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, Hq, 2, tokens};
  cuuint64_t strides[3] = {256, 128, (cuuint64_t)Hq * 256};
  cuuint32_t box[4] = {64, 8, 2, run};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace rdl

namespace rdl {

// Summaries s [rows, 128] fp32 (row stride 512 B) viewed as (32 columns, rows, 4 slices):
// one box of box_rows rows lands as 4 slices [box_rows][128 B] (columns 0-31, 32-63, ...),
// each with the 128-byte swizzle.  Rows past the end read as zeros.
inline bool make_tmap_f32_rows(CUtensorMap* map, const void* base, unsigned long long rows, unsigned box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {32, rows, 4};
  cuuint64_t strides[2] = {512, 128};
  cuuint32_t box[3] = {32, box_rows, 4};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Summaries in the split layout ([hi 128 | lo 128] bf16, 512 B per row) viewed as
// (64 columns, rows, 4 segments): one box of box_rows rows lands as 4 segments [box_rows][128 B]
// (hi 0-63, hi 64-127, lo 0-63, lo 64-127), each with the 128-byte swizzle.
inline bool make_tmap_split_rows(CUtensorMap* map, const void* base, unsigned long long rows, unsigned box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, rows, 4};
  cuuint64_t strides[2] = {512, 128};
  cuuint32_t box[3] = {64, box_rows, 4};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace rdl
