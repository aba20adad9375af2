// Tensor maps for the SSD kernels' operand tiles and the backward's dB / dC
// sums (host side). A map over a
// row-major [rows][groups][features] bf16 tensor with five dimensions
// (feature_lo 8, row_lo 8, feature_hi, group, row_hi) and a box of
// (8, 8, features / 8, 1, 16) delivers 128 rows of one group into shared
// memory in the no-swizzle core-matrix order
//   (row >> 3) * (features * 16) + (feature >> 3) * 128 + (row & 7) * 16 + (feature & 7) * 2,
// rows past the tensor zero-filled. The encoder comes from the driver
// through the runtime's entry-point query, so the library links no driver
// library; without it the kernels copy rows with cp.async.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>

namespace ssm {

typedef CUresult (*SsdTensorMapEncode)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                       const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                       CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                       CUtensorMapFloatOOBfill);

inline SsdTensorMapEncode ssd_tensor_map_encoder() {
  static std::atomic<SsdTensorMapEncode> fn{nullptr};
  static std::atomic<bool> tried{false};
  SsdTensorMapEncode f = fn.load(std::memory_order_acquire);
  if (!f && !tried.load(std::memory_order_acquire)) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f = reinterpret_cast<SsdTensorMapEncode>(ptr);
    fn.store(f, std::memory_order_release);
    tried.store(true, std::memory_order_release);
  }
  return f;
}

// rows must be a multiple of 8 (the caller's L is), base 16-byte aligned.
inline bool ssd_tile_map(SsdTensorMapEncode enc, CUtensorMap* m, const void* base, size_t rows, int groups,
                         int features) {
  const cuuint64_t dims[5] = {8, 8, (cuuint64_t)features / 8, (cuuint64_t)groups, (cuuint64_t)rows / 8};
  const cuuint64_t strides[4] = {(cuuint64_t)groups * features * 2, 16, (cuuint64_t)features * 2,
                                 (cuuint64_t)8 * groups * features * 2};
  const cuuint32_t box[5] = {8, 8, (cuuint32_t)features / 8, 1, 16};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A map over a [rows][groups][128] fp32 tensor for bulk reductions of boxes
// of 32 states x 128 rows of one group, staged in shared memory in the
// 128-byte swizzled order (16-byte chunk k of a box row r at k ^ (r & 7)).
inline bool ssd_sum_map(SsdTensorMapEncode enc, CUtensorMap* m, void* base, size_t rows, int groups) {
  const cuuint64_t dims[3] = {128, (cuuint64_t)groups, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {128 * 4, (cuuint64_t)groups * 128 * 4};
  const cuuint32_t box[3] = {32, 1, 128};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ssm
