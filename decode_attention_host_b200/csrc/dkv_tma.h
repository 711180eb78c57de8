// dkv_tma.h -- host-side encoding of the tensor maps the HBM split kernel
// copies its K/V tiles with (a pool viewed as rows of head_dim 16-bit
// elements; boxes of 16 rows x 64 elements with the 128-byte swizzle).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "dkv_kernels.cuh"

namespace dkv {

// cuTensorMapEncodeTiled, looked up once through the runtime (the library
// links no driver library); nullptr if the driver does not provide it.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    else
      cudaGetLastError();
  });
  return fn;
}

// Tensor map of a pool of `rows` token rows (blocks * kv heads * block size)
// of D 16-bit elements starting at `pool` (16-byte aligned): boxes of 16 rows,
// either whole plain rows (`plain`, the K pool) or 64-element halves with the
// 128-byte swizzle (the V pool).  A null pool or zero rows gives a zeroed map
// that no copy uses.  Returns false if the driver rejects the map.
inline bool encode_pool_map(CUtensorMap* map, const void* pool, long long rows, int D, bool plain) {
  *map = CUtensorMap{};
  if (!pool || rows <= 0) return true;
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {plain ? static_cast<cuuint32_t>(D) : 64u, static_cast<cuuint32_t>(kTileTokens)};
  const cuuint32_t estride[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(pool), dims, strides, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, plain ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dkv
