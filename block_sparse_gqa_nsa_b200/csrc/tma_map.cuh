// Host-side construction of the 3D TMA tensor maps the tcgen05 kernels load with.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace lsrm {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda)
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 3D bf16 map over a [rows][heads][D] tensor with a (D, box_heads, box_rows) box, swizzled to
// the row width (64-byte rows for D = 32, 128-byte rows for D = 64)
inline bool make_map(CUtensorMap* map, const void* base, int D, int heads, long long rows, int box_heads, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr || base == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle swz = D == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map over float4 rows [rows][heads][4 floats] (no swizzle) with a (4, box_heads, box_rows) box
inline bool make_map_rows(CUtensorMap* map, const void* base, int heads, long long rows, int box_heads, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr || base == nullptr) return false;
  cuuint64_t dims[3] = {4, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {16, (cuuint64_t)heads * 16};
  cuuint32_t box[3] = {4, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lsrm
