// Host-side construction of TMA tensor maps (CUtensorMap) for the chunk kernels.
//
// The driver entry point cuTensorMapEncodeTiled is looked up once through the
// runtime (cudaGetDriverEntryPoint), so the library needs no link-time
// dependency on libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

namespace kda {

using TensorMapEncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                            const cuuint64_t *, const cuuint64_t *,
                                            const cuuint32_t *, const cuuint32_t *,
                                            CUtensorMapInterleave, CUtensorMapSwizzle,
                                            CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline TensorMapEncodeTiledFn tensor_map_encoder() {
  static TensorMapEncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TensorMapEncodeTiledFn>(p);
  });
  return fn;
}

// Row-major matrix [rows][cols] of `esize`-byte elements with a row pitch of
// `pitch_elems` elements; tiles of box_rows x box_cols, no swizzle.  Reads
// outside the matrix (including negative row coordinates) return zeros.
inline bool encode_rows(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, size_t esize,
                        uint64_t rows, uint64_t cols, uint64_t pitch_elems, uint32_t box_rows,
                        uint32_t box_cols) {
  TensorMapEncodeTiledFn fn = tensor_map_encoder();
  if (fn == nullptr || rows == 0 || cols == 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_elems * esize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace kda
