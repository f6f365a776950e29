// Host-side TMA tensor-map encoding shared by the tensor-core kernels.
// cuTensorMapEncodeTiled is a driver-API call; it is resolved at run time
// through the runtime's entry-point query so that libsas links only against
// the CUDA runtime and loads on machines without a driver (symbol checks).
#include <cuda.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace sas {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return (EncodeTiledFn)p;
  }();
  return fn;
}

// Row-major bf16 [planes][rows_per_plane][d] viewed as a 3-D tensor with a
// {64, 64, 1} box, 128-byte swizzle and zero fill outside the extents.
bool make_tma_map_bf16_3d(CUtensorMap* map, const void* base, int d, int rows_per_plane,
                          int planes) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows_per_plane, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows_per_plane * d * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major fp32 [planes][rows_per_plane][d] as a 3-D tensor with a
// {box_d, box_rows, 1} box and no swizzle (reduce-add targets).
bool make_tma_map_f32_3d(CUtensorMap* map, const void* base, int d, int rows_per_plane,
                         int planes, int box_d, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows_per_plane, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)rows_per_plane * d * 4};
  const cuuint32_t box[3] = {(cuuint32_t)box_d, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sas
