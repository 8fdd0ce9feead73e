// vsa_tma.h -- host-side construction of the TMA tensor maps the kernels use
// (cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library needs no link against the driver library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace vsa {

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// [rows, d] bf16 viewed as (64 elements, 8 rows, d/64 halves, rows/8 groups):
// one box {64, 8, d/64, 8} is a whole 64-row block stored as
// [row group][d-half][8 rows][128 B], i.e. 1 KiB swizzle atoms with the
// d-halves of a row group side by side.
inline bool make_map4(CUtensorMap *m, const void *base, int64_t rows, int d) {
  EncodeFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {64, 8, static_cast<cuuint64_t>(d / 64),
                              static_cast<cuuint64_t>(rows / 8)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, 128,
                                 static_cast<cuuint64_t>(d) * 2 * 8};
  const cuuint32_t box[4] = {64, 8, static_cast<cuuint32_t>(d / 64), 8};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Raster [frames, H, W, d] bf16 (frames = B * heads * T) viewed as
// (64 elements, W columns, d/64 halves, H rows, frames): the box
// {64, 8, d/64, 8, 1} at (0, 8 px, 0, 8 py, frame) is the 8 x 8 patch
// (py, px) of one frame -- the 64 tokens of one fractal block, in-patch
// row-major -- stored in the same [patch row][d-half][8 tokens][128 B] order
// as the flattened map's box.  The fractal permutation is then done by the
// copy engine's addressing instead of by a separate pass over memory.
inline bool make_map_raster(CUtensorMap *m, const void *base, int64_t frames, int H, int W,
                            int d) {
  EncodeFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(d / 64),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(frames)};
  const cuuint64_t row = static_cast<cuuint64_t>(d) * 2;             // one token
  const cuuint64_t strides[4] = {row, 128, row * W, row * W * H};
  const cuuint32_t box[5] = {64, 8, static_cast<cuuint32_t>(d / 64), 8, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace vsa
