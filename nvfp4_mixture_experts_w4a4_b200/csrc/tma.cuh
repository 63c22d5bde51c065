// Tensor-map helpers shared by the tcgen05 kernels.
#pragma once

#include <cudaTypedefs.h>

#include "common.cuh"

namespace nvfp4moe {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// K-major NVFP4 code matrix [rows][K/2] bytes; box = 128 bytes (256 elements) x box_rows
// rows, 128-byte swizzle (the layout the UMMA shared-memory descriptors describe).
inline nvfp4moe_status make_code_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return fail(NVFP4MOE_CUDA_ERROR, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {cuuint64_t(K / 2), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(K / 2)};
  const cuuint32_t box[2] = {128u, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4MOE_CUDA_ERROR, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return NVFP4MOE_OK;
}

// fp32 matrix [rows][cols] (row pitch cols * 4 bytes), no swizzle, box = box_cols x box_rows:
// the tiles the down epilogue stores.  Rows past `rows` are clipped on store.
inline nvfp4moe_status make_f32_rows_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols, int box_cols,
                                         int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return fail(NVFP4MOE_CUDA_ERROR, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(cols * 4)};
  const cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4MOE_CUDA_ERROR, "cuTensorMapEncodeTiled (fp32 rows) failed (%d)", int(r));
  return NVFP4MOE_OK;
}

}  // namespace nvfp4moe
