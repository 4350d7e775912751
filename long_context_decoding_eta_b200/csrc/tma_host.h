// Host-side TMA tensor maps: the bf16 [rows, d] views the tcgen05 kernels load
// (K, V, queries; box of 64 columns x box_rows rows with 128-byte swizzle), the
// swizzled bf16 centroid view of the tensor-core screen, and plain 2-D views (the
// CUDA-core screens' metadata tiles).  The encoder is the driver's
// cuTensorMapEncodeTiled, looked up once through the runtime.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace eta {

using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

inline EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D view [rows, cols] of a bf16 tensor (cols 128 or 64; row stride 2 cols bytes).
inline bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows,
                     uint64_t cols = 128) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 2-D view of a bf16 tensor, `cols` x `rows` elements, row stride `row_bytes` (a
// multiple of 16); box 64 columns (128 bytes) x box_rows rows with 128-byte swizzle.
// Out-of-range elements of a box read as zero.
inline bool make_map_bf16_swz(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                              uint64_t row_bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {row_bytes};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// General 2-D map without swizzle: `cols` x `rows` elements of `dtype`, row stride
// `row_bytes` (a multiple of 16), box box_cols x box_rows; out-of-range elements
// of a box read as zero.
inline bool make_map_plain(CUtensorMap* m, const void* base, CUtensorMapDataType dtype,
                           uint64_t cols, uint64_t rows, uint64_t row_bytes, uint32_t box_cols,
                           uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dtype, 2, const_cast<void*>(base), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace eta
