// Host-side construction of TMA tensor maps (cuTensorMapEncodeTiled, fetched from the driver
// through the runtime so that the library links only against cudart).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D bf16 view: `rows` rows of `cols` elements, `row_bytes` apart, copied in 128-byte swizzled
// boxes of 64 columns x box_rows rows (out-of-range elements read as zero). Fails when the base
// or the row pitch is not 16-byte aligned or the driver rejects the shape.
inline bool make_bf16_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                          uint64_t row_bytes, uint32_t box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn || ((uintptr_t)base & 15) || (row_bytes & 15) || box_rows == 0 || box_rows > 256)
    return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace mla
