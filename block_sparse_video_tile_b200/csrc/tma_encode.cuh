// tma_encode.cuh -- host-side encoding of the TMA descriptors for Q, K, V.
//
// The driver's cuTensorMapEncodeTiled is reached through the runtime's
// driver-entry-point query, so the library needs no link against libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "vsa.h"
#include "vsa_geometry.cuh"

namespace vsa {

// ----------------------------------------------------------- TMA encoding
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B*H, T, Hh, W, d] bf16 viewed as a 5-D tensor (d innermost); box = 64
// channels x (tw, th, box_t) tokens, 128-byte swizzle, zero fill past edges.
inline int encode_qkv_map(CUtensorMap* m, const void* ptr, const Geom& g, int box_t, bool f16 = false) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return VSA_ERR_CUDA;
  const cuuint64_t e = 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(g.d), static_cast<cuuint64_t>(g.W),
                        static_cast<cuuint64_t>(g.Hh), static_cast<cuuint64_t>(g.T),
                        static_cast<cuuint64_t>(g.B) * g.H};
  cuuint64_t strides[4] = {e * g.d, e * g.d * g.W, e * g.d * g.W * g.Hh, e * g.d * g.W * g.Hh * g.T};
  cuuint32_t box[5] = {64u, static_cast<cuuint32_t>(g.tw), static_cast<cuuint32_t>(g.th),
                       static_cast<cuuint32_t>(box_t), 1u};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace vsa
