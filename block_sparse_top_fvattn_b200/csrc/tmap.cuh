// Host-side creation of TMA tensor maps (cuTensorMapEncodeTiled, looked up through the runtime's
// driver entry point so that the library needs no link-time libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace fv {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn lookup_encode_fn() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(p);
  return nullptr;
}

// Looked up once; the initialisation of a function-local static is thread-safe.
inline EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = lookup_encode_fn();
  return fn;
}

// A 3-D tensor [planes][rows][cols] (cols innermost, row stride `cols` elements of elem_bytes)
// read in boxes of 128 bytes of columns x box_rows rows with the 128-byte swizzle; rows past
// `rows` read as zeros and never reach the next plane.
inline bool make_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* base,
                        uint64_t cols, uint64_t rows, uint64_t planes, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)cols * elem_bytes, (cuuint64_t)rows * (cuuint64_t)cols * elem_bytes};
  cuuint32_t box[3] = {128 / elem_bytes, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [planes][rows][cols]: boxes of 64 columns.
inline bool make_map_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t planes,
                             uint32_t box_rows) {
  return make_map_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, cols, rows, planes, box_rows);
}

// 8-bit integers [planes][rows][cols]: boxes of 128 columns.
inline bool make_map_i8_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t planes,
                           uint32_t box_rows) {
  return make_map_3d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, cols, rows, planes, box_rows);
}

}  // namespace fv
