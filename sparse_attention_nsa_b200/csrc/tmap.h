// tmap.h -- host-side creation of TMA tensor maps for the tensor-core
// kernels (driver entry point looked up once through the runtime).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

namespace nsa {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  });
  return fn;
}

// 3-D bf16 view (64 head dims, heads, rows) of a row-major [rows, heads, 64]
// tensor, loaded in (64, box_h, box_rows) boxes with the 128-byte swizzle;
// reads outside the tensor return zeros.  rows must be >= 1.
inline bool make_tmap_bf16(CUtensorMap* map, const void* base, int heads, long rows, int box_h,
                           int box_rows) {
  auto fn = tmap_encode_fn();
  if (!fn || rows < 1) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {128, (cuuint64_t)heads * 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_h, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace nsa
