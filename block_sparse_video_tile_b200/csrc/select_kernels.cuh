// select_kernels.cuh -- tile selection: mean-pooling, tile scores, top-k.
//
// FastVideo VSA user guide (intro): for every query block, VSA scores the
// key/value blocks and keeps the top-k ("Wan top-k behavior": top-k counts
// key/value blocks per query block).  Scores are dot products of the tiles'
// mean-pooled Q and K.  fastbsa page ("How it works"): selection stays in
// shared memory instead of round-tripping a score matrix through HBM.
//
// Two kernels:
//   pool_kernel   HBM-bound: reads every Q and K byte once, writes the per-tile
//                 means (float32 [2, B*H, nT, d]) to the caller's workspace.
//   score_topk_kernel: per (head, block of query tiles) computes the score
//                 rows into shared memory (float32 FMA in a fixed order) and
//                 selects each row's top-k exactly; writes ascending idx.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include <cuda.h>

#include "vsa_geometry.cuh"
#include "vsa_ptx.cuh"

namespace vsa {

constexpr int kPoolThreads = 256;

// One CTA per (tile j, head bh, tensor z in {Q, K}).  The whole tile is one
// 5-D TMA box per 64-channel slab (the same [B*H, T, Hh, W, d] view the
// attend kernel uses), so a 256-token tile of d = 128 puts 64 KB in flight
// per CTA without using registers; positions past the grid edge arrive as
// zeros and add nothing to the sums.  Threads then sum 16-byte chunks down the
// rows in a fixed order (deterministic) and divide by the tile's valid count.
// Dynamic shared memory: box (slabs x vol x 128 B, 1024-aligned) | partial sums | mbarrier.
template <int D, bool F16>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                            const __grid_constant__ CUtensorMap tmK, Geom g,
                                                            float* __restrict__ pooled, unsigned int* err) {
  constexpr int kSlabs = D / 64;
  constexpr int TPR = D / 8;                 // threads per row (one 16-byte chunk each)
  constexpr int RP = kPoolThreads / TPR;     // row groups
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sp = smem_raw + (base - raw);
  const int vol = g.vol;
  const int box_bytes = vol * 128;
  float* part = reinterpret_cast<float*>(sp + kSlabs * box_bytes);     // [RP][D]
  const uint32_t bar = base + kSlabs * box_bytes + RP * D * 4;

  const int j = blockIdx.x;
  const int bh = blockIdx.y;
  const int z = blockIdx.z;
  const TileCoord c = tile_coord(g, j);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kSlabs * box_bytes));
    for (int sl = 0; sl < kSlabs; ++sl)
      tma_load_5d(base + sl * box_bytes, z == 0 ? static_cast<const void*>(&tmQ) : static_cast<const void*>(&tmK),
                  bar, sl * 64, c.bx * g.tw, c.by * g.th, c.bt * g.tt, bh);
  }
  // let the score kernel's launch begin while this grid drains
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __syncthreads();
  const bool ok = mbar_wait(bar, 0, nullptr, err);

  const int cc = threadIdx.x % TPR;          // 16-byte chunk of the row: slab cc/8, chunk cc%8
  const int rg = threadIdx.x / TPR;
  const unsigned char* slab = sp + (cc / 8) * box_bytes;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (ok) {
#pragma unroll 4
    for (int r = rg; r < vol; r += RP) {
      const uint4 u = *reinterpret_cast<const uint4*>(slab + r * 128 + (((cc % 8) ^ (r & 7)) << 4));
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_elem2<F16>(w4[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg * D + cc * 8 + e] = acc[e];
  __syncthreads();
  int vt, vy, vx;
  tile_extent(g, c, vt, vy, vx);
  const float cnt = static_cast<float>(vt * vy * vx);
  for (int col = threadIdx.x; col < D; col += kPoolThreads) {
    float sum = 0.f;
#pragma unroll 8
    for (int i = 0; i < RP; ++i) sum += part[i * D + col];
    pooled[((static_cast<size_t>(z) * g.B * g.H + bh) * g.nT + j) * D + col] = sum / cnt;
  }
}

template <int D>
inline size_t pool_smem_bytes(const Geom& g) {
  return static_cast<size_t>(D / 64) * g.vol * 128 + (kPoolThreads / (D / 8)) * D * 4 + 16 + 1024;
}

constexpr int kScoreThreads = 256;  // 8 warps

// Larger float -> larger unsigned key (total order; -0 < +0, scores are
// canonicalised so -0 does not occur).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exact top-k of one row of order keys by one warp, keys held in registers
// (lane l holds tiles l, l + 32, ...).  The topk-th largest key T is found
// bit by bit from the top: T keeps a bit when at least topk keys are >= T
// with that bit set (a warp-wide count per bit, no shared-memory atomics).
// Every key above T is taken, then the keys equal to T in ascending tile
// order until topk are taken (ties go to the lower tile index); indices are
// written in ascending order.  Order keys of finite scores are never 0, so 0
// marks the padding slots.
template <int MAXE>
__device__ __forceinline__ void bsearch_topk_row(const uint32_t* kr, int nT, int topk, int32_t* out) {
  const int lane = threadIdx.x % 32;
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t key[MAXE];
#pragma unroll
  for (int e = 0; e < MAXE; ++e) {
    const int j = lane + 32 * e;
    key[e] = (j < nT) ? kr[j] : 0u;
  }
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = T | (1u << b);
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < MAXE; ++e) c += (key[e] >= cand) ? 1u : 0u;
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= static_cast<uint32_t>(topk)) T = cand;
  }
  uint32_t gt = 0;
#pragma unroll
  for (int e = 0; e < MAXE; ++e) gt += (key[e] > T) ? 1u : 0u;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int want_eq = topk - static_cast<int>(gt);
  int base = 0, eq_seen = 0;
#pragma unroll
  for (int e = 0; e < MAXE; ++e) {
    if (32 * e >= nT) break;
    const bool gtb = key[e] > T;
    const bool eqb = key[e] == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eqb);
    const bool take = gtb || (eqb && eq_seen + __popc(eqm & lt_mask) < want_eq);
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (take) out[base + __popc(tm & lt_mask)] = lane + 32 * e;
    base += __popc(tm);
    eq_seen += __popc(eqm);
  }
}

// Tile scores and top-k.  One CTA takes R query tiles of one head (R = 8 when
// the head has at most 256 tiles, else 16).  Their pooled Q means and the
// pooled K means, in chunks of up to 64 key tiles (rows padded to d + 4
// floats), are copied to shared memory with vector loads.  Thread t =
// (quarter, j) forms, for key tile j of the chunk and all R query tiles, the
// partial dot product over its quarter of the d channels: the padded rows make
// the key reads of a quarter-warp hit 8 different bank groups, and the query
// reads are warp-wide broadcasts.  The four partial sums are added in a fixed
// order (deterministic); the score rows stay in shared memory as order keys,
// and one warp per row selects its top-k.  Shared memory stays under 76 KB
// for up to 256 tiles, so three CTAs fit on an SM.
// Dynamic shared memory: qb[R][D] | kb[min(nT,64)][D+4] | part[4][R][64] | keys[R][nT]
constexpr int kScoreChunk = 64;
constexpr int kScoreSplit = kScoreThreads / kScoreChunk;   // d split in 4 parts

template <int D, int R>
__global__ void __launch_bounds__(kScoreThreads) score_topk_kernel(Geom g, const float* __restrict__ pooled,
                                                                   int topk, int32_t* __restrict__ idx) {
  constexpr int KS = D + 4;                 // padded key-mean row (floats)
  constexpr int C4 = D / 4;
  constexpr int PART4 = D / 4 / kScoreSplit;  // float4 chunks per part of a row
  constexpr int MAXE = (R == 8) ? 8 : 48;   // keys per lane in the top-k (nT <= 256 / <= 1536)
  // the pooled means are written by the previous grid: wait for it
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int nT = g.nT;
  const int chunk = min(nT, kScoreChunk);
  float* qb = reinterpret_cast<float*>(smem_raw);
  float* kb = qb + R * D;
  float* part = kb + chunk * KS;
  uint32_t* keys = reinterpret_cast<uint32_t*>(part + kScoreSplit * R * kScoreChunk);

  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * R;
  const int nrows = min(R, nT - row0);
  const size_t BH = static_cast<size_t>(g.B) * g.H;
  const float4* qp = reinterpret_cast<const float4*>(pooled + (static_cast<size_t>(bh) * nT + row0) * D);
  const float4* kp = reinterpret_cast<const float4*>(pooled + ((BH + bh) * nT) * D);

#pragma unroll 4
  for (int e = threadIdx.x; e < R * C4; e += kScoreThreads)
    reinterpret_cast<float4*>(qb)[e] = (e / C4 < nrows) ? __ldg(qp + e) : make_float4(0.f, 0.f, 0.f, 0.f);

  const int j = threadIdx.x % kScoreChunk;
  const int quarter = threadIdx.x / kScoreChunk;
  for (int c0 = 0; c0 < nT; c0 += kScoreChunk) {
    const int ncol = min(kScoreChunk, nT - c0);
    if (c0 > 0) __syncthreads();   // the previous chunk's partial sums are consumed
#pragma unroll 8
    for (int e = threadIdx.x; e < ncol * C4; e += kScoreThreads) {
      const int r = e / C4, c = e % C4;
      *reinterpret_cast<float4*>(kb + r * KS + 4 * c) = __ldg(kp + static_cast<size_t>(c0) * C4 + e);
    }
    __syncthreads();
    if (j < ncol) {
      float acc[R];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = 0.f;
      const float4* krow = reinterpret_cast<const float4*>(kb + j * KS) + quarter * PART4;
      const float4* qrow = reinterpret_cast<const float4*>(qb) + quarter * PART4;
#pragma unroll 4
      for (int i = 0; i < PART4; ++i) {
        const float4 kv = krow[i];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float4 qv = qrow[r * C4 + i];
          acc[r] = fmaf(qv.x, kv.x, acc[r]);
          acc[r] = fmaf(qv.y, kv.y, acc[r]);
          acc[r] = fmaf(qv.z, kv.z, acc[r]);
          acc[r] = fmaf(qv.w, kv.w, acc[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) part[(quarter * R + r) * kScoreChunk + j] = acc[r];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < R * ncol; e += kScoreThreads) {
      const int r = e / ncol, c = e % ncol;
      const float sc = (part[r * kScoreChunk + c] + part[(R + r) * kScoreChunk + c]) +
                       (part[(2 * R + r) * kScoreChunk + c] + part[(3 * R + r) * kScoreChunk + c]);
      keys[r * nT + c0 + c] = order_key(sc + 0.f);
    }
  }
  __syncthreads();

  const int warp = threadIdx.x / 32;
  for (int r = warp; r < nrows; r += kScoreThreads / 32) {
    int32_t* out = idx + (static_cast<size_t>(bh) * nT + row0 + r) * topk;
    if (MAXE > 24 && nT <= 32 * 24)   // fewer keys per lane: a shorter unrolled count loop
      bsearch_topk_row<(MAXE > 24 ? 24 : MAXE)>(keys + r * nT, nT, topk, out);
    else
      bsearch_topk_row<MAXE>(keys + r * nT, nT, topk, out);
  }
}

template <int D, int R>
inline size_t score_smem_bytes(const Geom& g) {
  const size_t chunk = static_cast<size_t>(min(g.nT, kScoreChunk));
  return sizeof(float) * (static_cast<size_t>(R) * D + chunk * (D + 4) + kScoreSplit * static_cast<size_t>(R) * kScoreChunk) +
         sizeof(uint32_t) * (static_cast<size_t>(R) * g.nT);
}

}  // namespace vsa
