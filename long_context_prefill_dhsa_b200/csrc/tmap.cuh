// TMA tensor maps of the attention kernels: a [rows, 128] bf16 row-major
// matrix (Q, K or V with the (batch, head, token) rows flattened) read in
// boxes of 64 columns x `box_rows` rows with 128-byte swizzle, so that each
// box lands as one K-major (or M/N-major) tcgen05 operand block.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace dhsa {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no
// link-time dependency on libcuda).
inline EncodeTiledFn tmap_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Rows past `rows` read as zeros.
inline bool make_rows_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, long long rows, int box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A view of every `step`-th row of a [rows_total, kHeadDim] bf16 tensor,
// starting at `base`: view row y is base row step*y. Rows past `rows` read
// as zeros.
inline bool make_rows_view_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, long long rows, int step,
                               int box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2 * step};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Work lists of the two attention kernels (built on the device by
// launch_build_items). Long items are (b, hq, chunk, 128-row tile index),
// short items (b, hq, chunk, first row of the tile within the chunk).
struct AttnWork {
  int4* items_long;
  int* n_long;
  int* counter_long;     // next unassigned long item, zeroed by the builder
  long long cap_long;    // capacity (0: no long items)
  int4* items_short;
  int* n_short;
  int* counter_short;
  long long cap_short;
};

}  // namespace dhsa
