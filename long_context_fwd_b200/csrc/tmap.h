// tmap.h -- host-side TMA tensor-map encoding for the kernels of this library.
// cuTensorMapEncodeTiled is fetched through the runtime's driver entry-point
// query so the library does not link libcuda directly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Tensor map over a contiguous [planes][rows][cols] array (cols innermost),
// box = {box_cols, box_rows, 1}, 128-byte swizzle, zero fill out of bounds.
// box_cols * elem_bytes must be 128 (one swizzle row).  Returns false on error.
inline bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         uint32_t elem_bytes, uint64_t cols, uint64_t rows, uint64_t planes,
                         uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, planes};
  cuuint64_t strides[2] = {cols * elem_bytes, cols * rows * elem_bytes};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over a 4-D array [b][h][t][col] with arbitrary element strides
// for the t, h and b dimensions (cols contiguous): box = box_cols columns x
// box_rows tokens of one (b, h), 128-byte swizzle, zero fill out of bounds.
// The three outer dimensions are put in the map in increasing stride order;
// *slots receives where t, h and b went (2 bits each, values 1..3: t | h << 2
// | b << 4).  box_cols * elem_bytes must be 128.  Returns false on error.
inline bool make_tmap_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         uint32_t elem_bytes, uint64_t cols, const uint64_t ext[3],
                         const uint64_t stride_elems[3], uint32_t box_cols, uint32_t box_rows,
                         int* slots) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  int order[3] = {0, 1, 2};  // 0 = t, 1 = h, 2 = b
  for (int i = 1; i < 3; ++i)
    for (int j = i; j > 0 && stride_elems[order[j]] < stride_elems[order[j - 1]]; --j) {
      const int tmp = order[j];
      order[j] = order[j - 1];
      order[j - 1] = tmp;
    }
  cuuint64_t dims[4] = {cols, 0, 0, 0};
  cuuint64_t strides[3];
  cuuint32_t box[4] = {box_cols, 1, 1, 1};
  int packed = 0;
  for (int i = 0; i < 3; ++i) {
    const int d = order[i];
    dims[1 + i] = ext[d];
    strides[i] = stride_elems[d] * elem_bytes;
    if (d == 0) box[1 + i] = box_rows;
    packed |= (1 + i) << (2 * d);
  }
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  *slots = packed;
  return true;
}

}  // namespace la
