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

// One side's Q, K or V viewed as a 5-D tensor, d innermost: [B, H, N, d] as
// (d, W, Hh, T, B*H) with box (64, tw, th, box_t, 1); [B, N, H, d] as
// (d, H, W, Hh, B*T) with box (64, 1, tw, th, box_t).  Either box lands in
// shared memory as box_t*th*tw rows of 64 channels in raster order, 128-byte
// swizzle, zero fill past the edges (in the second view a box that runs past
// T reads the next batch's first frames instead: consumers mask those rows).
inline int encode_qkv_map(CUtensorMap* m, const void* ptr, const Geom& g, int box_t, bool f16 = false) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return VSA_ERR_CUDA;
  const cuuint64_t e = 2;
  const cuuint64_t d = static_cast<cuuint64_t>(g.d), W = static_cast<cuuint64_t>(g.W),
                   Hh = static_cast<cuuint64_t>(g.Hh), T = static_cast<cuuint64_t>(g.T),
                   B = static_cast<cuuint64_t>(g.B), H = static_cast<cuuint64_t>(g.H);
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5];
  if (g.layout == 1) {
    const cuuint64_t dv[5] = {d, H, W, Hh, B * T};
    const cuuint64_t sv[4] = {e * d, e * d * H, e * d * H * W, e * d * H * W * Hh};
    const cuuint32_t bv[5] = {64u, 1u, static_cast<cuuint32_t>(g.tw), static_cast<cuuint32_t>(g.th),
                              static_cast<cuuint32_t>(box_t)};
    for (int i = 0; i < 5; ++i) { dims[i] = dv[i]; box[i] = bv[i]; }
    for (int i = 0; i < 4; ++i) strides[i] = sv[i];
  } else {
    const cuuint64_t dv[5] = {d, W, Hh, T, B * H};
    const cuuint64_t sv[4] = {e * d, e * d * W, e * d * W * Hh, e * d * W * Hh * T};
    const cuuint32_t bv[5] = {64u, static_cast<cuuint32_t>(g.tw), static_cast<cuuint32_t>(g.th),
                              static_cast<cuuint32_t>(box_t), 1u};
    for (int i = 0; i < 5; ++i) { dims[i] = dv[i]; box[i] = bv[i]; }
    for (int i = 0; i < 4; ++i) strides[i] = sv[i];
  }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

// The output map: the query side's boxes, with dimensions that keep every
// box inside its own batch, so that a store clips the rows outside the grid.
// [B, H, N, d] as the Q map (T is a dimension of its own); [B, N, H, d]:
// (H * d channels, W, Hh, T, B) -- a head's d channels are contiguous and the
// heads of a token follow each other, so the box's channel coordinate is
// h * d + c.
inline int encode_o_map(CUtensorMap* m, void* ptr, const Geom& g, int box_t, bool f16 = false) {
  if (g.layout != 1) return encode_qkv_map(m, ptr, g, box_t, f16);
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return VSA_ERR_CUDA;
  const cuuint64_t e = 2;
  const cuuint64_t d = static_cast<cuuint64_t>(g.d), W = static_cast<cuuint64_t>(g.W),
                   Hh = static_cast<cuuint64_t>(g.Hh), T = static_cast<cuuint64_t>(g.T),
                   B = static_cast<cuuint64_t>(g.B), H = static_cast<cuuint64_t>(g.H);
  cuuint64_t dims[5] = {H * d, W, Hh, T, B};
  cuuint64_t strides[4] = {e * d * H, e * d * H * W, e * d * H * W * Hh, e * d * H * W * Hh * T};
  cuuint32_t box[5] = {64u, static_cast<cuuint32_t>(g.tw), static_cast<cuuint32_t>(g.th),
                       static_cast<cuuint32_t>(box_t), 1u};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, ptr, dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

}  // namespace vsa
