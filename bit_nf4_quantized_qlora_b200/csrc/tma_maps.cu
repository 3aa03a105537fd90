// Host-side TMA tensor-map encoding (cuTensorMapEncodeTiled through the
// runtime's driver entry point, so the library does not link libcuda).
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace qlora {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 2D map over a row-major [outer x inner] tensor with a row pitch in bytes.
// Out-of-range elements of a box read as zero.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool encode_f32_slab_map(CUtensorMap *m, const float *ptr, int64_t slabs, int64_t rows, int64_t cols,
                         uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(slabs)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 4u, static_cast<cuuint64_t>(rows * cols) * 4u};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_bf16_map(CUtensorMap *m, const uint16_t *ptr, int64_t rows, int64_t cols, uint32_t box_cols,
                     uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                  static_cast<uint64_t>(cols) * 2u, box_cols, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_f32_map(CUtensorMap *m, const float *ptr, int64_t rows, int64_t cols, uint32_t box_cols,
                    uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ptr, static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                  static_cast<uint64_t>(cols) * 4u, box_cols, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_codes_map(CUtensorMap *m, const uint8_t *ptr, int64_t rows, int64_t row_bytes, uint32_t box_bytes,
                      uint32_t box_rows, bool swizzle128) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, ptr, static_cast<uint64_t>(row_bytes),
                  static_cast<uint64_t>(rows), static_cast<uint64_t>(row_bytes), box_bytes, box_rows,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace qlora
