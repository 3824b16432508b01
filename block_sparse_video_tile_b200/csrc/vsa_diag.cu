// vsa_diag.cu -- bring-up checks for the building blocks of the attend kernel,
// built as libvsa_diag.so and used only by the tests.
//
//   vsa_diag_tma_box  one 5-D TMA box of a [B*H, T, Hh, W, d] tensor into
//                     shared memory, copied out byte for byte (still in the
//                     128-byte-swizzled layout) so the host can check the
//                     tile index map, the zero fill and the swizzle.
//   vsa_diag_mma_ss   C[128x128] = A[128xD] * B[128xD]^T with both operands
//                     in 128B-swizzled K-major shared memory (the S = Q K^T step).
//   vsa_diag_mma_ts   O[128xD] = P[128x128] * V[128xD] with P in TMEM (two
//                     bf16 per column) and V in 128B-swizzled MN-major shared
//                     memory (the O += P V step).
//   vsa_diag_exp2     the FMA-pipe and multi-function-unit 2^x of the softmax.
//   vsa_diag_wait_timeout  a bounded mbarrier wait that nothing completes:
//                     it must end with a timeout in the error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "vsa.h"
#include "tma_encode.cuh"
#include "vsa_geometry.cuh"
#include "vsa_ptx.cuh"

namespace vsa {
__device__ unsigned int g_diag_error = 0u;

// byte offset of 16-byte chunk c of row r in a 128B-swizzled slab
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__global__ void diag_tma_kernel(const __grid_constant__ CUtensorMap tm, int slabs, int box_rows, int c1, int c2,
                                int c3, int c4, uint4* out, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sp = smem_raw + (base - raw);
  const uint32_t bar = base + 2 * 16384;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(slabs * box_rows * 128));
    for (int sl = 0; sl < slabs; ++sl) tma_load_5d(base + sl * 16384, &tm, bar, sl * 64, c1, c2, c3, c4);
  }
  mbar_wait(bar, 0, nullptr, err);
  const uint4* src = reinterpret_cast<const uint4*>(sp);
  for (int sl = 0; sl < slabs; ++sl)
    for (int e = threadIdx.x; e < box_rows * 8; e += blockDim.x)
      out[sl * box_rows * 8 + e] = src[sl * 1024 + e];
}

template <int D>
__global__ void diag_mma_ss_kernel(const uint4* A, const uint4* B, float* C, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sp = smem_raw + (base - raw);
  constexpr int kSlabs = D / 64;
  const uint32_t sA = base, sB = base + kSlabs * 16384, bar = base + 2 * kSlabs * 16384;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sp + 2 * kSlabs * 16384 + 8);
  // software-swizzled fill: row r, chunk c (8 bf16) of slab sl
  for (int e = threadIdx.x; e < 128 * (D / 8); e += blockDim.x) {
    const int r = e / (D / 8), cc = e % (D / 8), sl = cc / 8, c = cc % 8;
    *reinterpret_cast<uint4*>(sp + sl * 16384 + sw128(r, c)) = A[e];
    *reinterpret_cast<uint4*>(sp + kSlabs * 16384 + sl * 16384 + sw128(r, c)) = B[e];
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(tslot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (threadIdx.x == 0) {
    constexpr uint32_t id = idesc_bf16_f32(128, 128, false);
    for (int kk = 0; kk < D / 16; ++kk) {
      const int sl = kk / 4, koff = (kk % 4) * 32;
      mma_ss(tmem, smem_desc_sw128(sA + sl * 16384 + koff, 16, 1024),
             smem_desc_sw128(sB + sl * 16384 + koff, 16, 1024), id, kk > 0 ? 1u : 0u);
    }
    mma_commit(bar);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, nullptr, err));
  tc_fence_after();
  const int w = threadIdx.x / 32, r = threadIdx.x;
  for (int c4 = 0; c4 < 4; ++c4) {
    uint32_t v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(w * 32) << 16) + 32u * c4, v);
    tmem_wait_ld();
    if (ok)
      for (int e = 0; e < 32; ++e) C[r * 128 + 32 * c4 + e] = __uint_as_float(v[e]);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <int D>
__global__ void diag_mma_ts_kernel(const uint32_t* P, const uint4* V, float* O, unsigned int* err) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sp = smem_raw + (base - raw);
  constexpr int kSlabs = D / 64;
  const uint32_t sV = base, bar = base + kSlabs * 16384;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sp + kSlabs * 16384 + 8);
  // V [128 kv][D]: slab sl holds columns [64 sl, 64 sl + 64) of every kv row
  for (int e = threadIdx.x; e < 128 * (D / 8); e += blockDim.x) {
    const int r = e / (D / 8), cc = e % (D / 8), sl = cc / 8, c = cc % 8;
    *reinterpret_cast<uint4*>(sp + sl * 16384 + sw128(r, c)) = V[e];
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(tslot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const int w = threadIdx.x / 32, r = threadIdx.x;
  const uint32_t lane_base = static_cast<uint32_t>(w * 32) << 16;
  {  // P row r (64 packed bf16 pairs) -> TMEM columns [0, 64)
    uint32_t v[32];
    for (int e = 0; e < 32; ++e) v[e] = P[r * 64 + e];
    tmem_st32(tmem + lane_base, v);
    for (int e = 0; e < 32; ++e) v[e] = P[r * 64 + 32 + e];
    tmem_st32(tmem + lane_base + 32, v);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    constexpr uint32_t id = idesc_bf16_f32(128, D, true);
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(tmem + 128, tmem + 8u * kk, smem_desc_sw128(sV + kk * 2048, 16384, 1024), id, kk > 0 ? 1u : 0u);
    mma_commit(bar);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, nullptr, err));
  tc_fence_after();
  for (int c4 = 0; c4 < D / 32; ++c4) {
    uint32_t v[32];
    tmem_ld32(tmem + lane_base + 128 + 32u * c4, v);
    tmem_wait_ld();
    if (ok)
      for (int e = 0; e < 32; ++e) O[r * D + 32 * c4 + e] = __uint_as_float(v[e]);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void diag_exp2_kernel(const float* x, float* y_poly, float* y_mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 >= n + 1) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  float p0, p1;
  exp2_poly_pair(f2_pack(a, b), p0, p1);
  y_poly[i] = p0;
  y_mufu[i] = ex2_approx(a);
  if (i + 1 < n) {
    y_poly[i + 1] = p1;
    y_mufu[i + 1] = ex2_approx(b);
  }
}

// A wait that nothing ever completes: the bounded wait must give up after its
// time limit, record the timeout in the error word and let the kernel return.
__global__ void diag_wait_timeout_kernel(unsigned int* err, int* returned) {
  __shared__ __align__(8) unsigned long long bar_storage;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(bar, 0, nullptr, err);   // nobody arrives
  if (threadIdx.x == 0) *returned = ok ? 2 : 1;
}

static unsigned int* diag_err() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_diag_error) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}

}  // namespace vsa

using namespace vsa;

extern "C" {

// Loads the box of tile j (t offset toff inside the tile, box t-extent box_t)
// of head bh from x [B*H, T, Hh, W, d] and writes the raw shared-memory bytes
// (d/64 slabs of box rows x 128 bytes, 128B-swizzled) to out.
int vsa_diag_tma_box(const vsa_shape* s, const void* x, int32_t box_t, int32_t j, int32_t toff, int32_t bh,
                     void* out, void* stream) {
  Geom g;
  g.B = s->B; g.H = s->H; g.T = s->T; g.Hh = s->Hh; g.W = s->W; g.d = s->d;
  g.tt = s->tt; g.th = s->th; g.tw = s->tw;
  g.nTt = ceil_div(g.T, g.tt); g.nTy = ceil_div(g.Hh, g.th); g.nTx = ceil_div(g.W, g.tw);
  g.nT = g.nTt * g.nTy * g.nTx;
  CUtensorMap m;
  int rc = encode_qkv_map(&m, x, g, box_t);
  if (rc != VSA_OK) return rc;
  const TileCoord c = tile_coord(g, j);
  const int box_rows = box_t * g.th * g.tw;
  const int smem = 2 * 16384 + 64 + 1024;
  cudaFuncSetAttribute(diag_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  diag_tma_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      m, g.d / 64, box_rows, c.bx * g.tw, c.by * g.th, c.bt * g.tt + toff, bh, static_cast<uint4*>(out), diag_err());
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int vsa_diag_mma_ss(const void* A, const void* B, int32_t d, float* C, void* stream) {
  const int smem = 2 * (d / 64) * 16384 + 64 + 1024;
  if (d == 128) {
    cudaFuncSetAttribute(diag_mma_ss_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    diag_mma_ss_kernel<128><<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(A), static_cast<const uint4*>(B), C, diag_err());
  } else if (d == 64) {
    cudaFuncSetAttribute(diag_mma_ss_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    diag_mma_ss_kernel<64><<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(A), static_cast<const uint4*>(B), C, diag_err());
  } else {
    return VSA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int vsa_diag_mma_ts(const void* P, const void* V, int32_t d, float* O, void* stream) {
  const int smem = (d / 64) * 16384 + 64 + 1024;
  if (d == 128) {
    cudaFuncSetAttribute(diag_mma_ts_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    diag_mma_ts_kernel<128><<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint32_t*>(P), static_cast<const uint4*>(V), O, diag_err());
  } else if (d == 64) {
    cudaFuncSetAttribute(diag_mma_ts_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    diag_mma_ts_kernel<64><<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint32_t*>(P), static_cast<const uint4*>(V), O, diag_err());
  } else {
    return VSA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// 2^x of n floats by the FMA-pipe polynomial (y_poly) and by ex2.approx (y_mufu).
int vsa_diag_exp2(const float* x, float* y_poly, float* y_mufu, int32_t n, void* stream) {
  const int pairs = (n + 1) / 2;
  diag_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_mufu, n);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// Launches one CTA whose only wait can never complete; *returned becomes 1
// once the bounded wait has given up.
int vsa_diag_wait_timeout(int32_t* returned, void* stream) {
  diag_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(diag_err(), returned);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

int vsa_diag_error(uint32_t* code) {
  if (cudaDeviceSynchronize() != cudaSuccess) return VSA_ERR_CUDA;
  unsigned int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_diag_error, sizeof(h)) != cudaSuccess) return VSA_ERR_CUDA;
  *code = h;
  const unsigned int z = 0;
  cudaMemcpyToSymbol(g_diag_error, &z, sizeof(z));
  return VSA_OK;
}

}  // extern "C"
