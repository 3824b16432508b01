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
//                 runs an exact radix select per row; writes ascending idx.
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
template <int D>
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
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
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
constexpr int kScoreChunk = 64;     // key tiles per shared-memory chunk
constexpr int kKtStride = kScoreChunk + 1;  // padded row of the transposed chunk

// Larger float -> larger unsigned key (total order; -0 < +0, scores are
// canonicalised so -0 does not occur).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exact top-k of one row of order keys by one warp: a 4-pass 8-bit radix
// select finds the topk-th largest key; every larger key and the first equal
// keys (lowest tile index first) are then written in ascending tile order.
__device__ __forceinline__ void radix_topk_row(const uint32_t* kr, int nT, int topk, uint32_t* hist,
                                               int32_t* out) {
  const int lane = threadIdx.x % 32;
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t prefix = 0, pmask = 0;
  int want = topk;  // rank (1-based) of the threshold among remaining candidates
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int jx = lane; jx < nT; jx += 32) {
      const uint32_t u = kr[jx];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l owns bins 255-8l .. 248-8l (descending digit order)
    uint32_t cnt8[8];
    uint32_t tot = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cnt8[e] = hist[255 - 8 * lane - e];
      tot += cnt8[e];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    uint32_t above = incl - tot;  // candidates with a larger digit than my bins
    int found_digit = -1;
    uint32_t found_above = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (found_digit < 0 && above < static_cast<uint32_t>(want) &&
          above + cnt8[e] >= static_cast<uint32_t>(want)) {
        found_digit = 255 - 8 * lane - e;
        found_above = above;
      }
      above += cnt8[e];
    }
    const uint32_t who = __ballot_sync(0xffffffffu, found_digit >= 0);
    const int src = __ffs(who) - 1;
    found_digit = __shfl_sync(0xffffffffu, found_digit, src);
    found_above = __shfl_sync(0xffffffffu, found_above, src);
    want -= static_cast<int>(found_above);
    prefix |= static_cast<uint32_t>(found_digit) << shift;
    pmask |= 255u << shift;
    __syncwarp();
  }
  // prefix is the topk-th largest key; take every larger key and the first
  // `want` keys equal to it (lowest tile index first), in ascending order.
  int base = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nT; j0 += 32) {
    const int jx = j0 + lane;
    const uint32_t u = (jx < nT) ? kr[jx] : 0u;
    const bool gt = (jx < nT) && (u > prefix);
    const bool eq = (jx < nT) && (u == prefix);
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && (eq_seen + __popc(eqm & lt_mask)) < want);
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (take) out[base + __popc(tm & lt_mask)] = jx;
    base += __popc(tm);
    eq_seen += __popc(eqm);
  }
}

// R query tiles per CTA (4 or 16: fewer rows give more CTAs when nT is small,
// more rows amortise the key-mean reads when nT is large).
// Dynamic shared memory: qb[R][D] | kT[D][CH+1] | keys[R][nT] (uint32) | hist[8][256]
template <int D, int R>
__global__ void __launch_bounds__(kScoreThreads) score_topk_kernel(Geom g, const float* __restrict__ pooled,
                                                                   int topk, int32_t* __restrict__ idx) {
  constexpr int kScoreRows = R;
  constexpr int RPT = R / 4;               // rows per thread in the score phase
  // wait until the pooling grid has finished and its writes are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qb = reinterpret_cast<float*>(smem_raw);
  float* kT = qb + kScoreRows * D;
  uint32_t* keys = reinterpret_cast<uint32_t*>(kT + D * kKtStride);
  uint32_t* hist_all = keys + kScoreRows * g.nT;

  const int nT = g.nT;
  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * kScoreRows;
  const int nrows = min(kScoreRows, nT - row0);
  const size_t BH = static_cast<size_t>(g.B) * g.H;
  const float* qp = pooled + (static_cast<size_t>(bh) * nT) * D;
  const float* kp = pooled + ((BH + bh) * nT) * D;

  for (int e = threadIdx.x; e < kScoreRows * D; e += kScoreThreads) {
    const int r = e / D;
    qb[e] = (r < nrows) ? qp[static_cast<size_t>(row0 + r) * D + (e % D)] : 0.f;
  }

  // score phase: thread -> (column jj, RPT consecutive rows)
  const int jj = threadIdx.x % kScoreChunk;
  const int rg = threadIdx.x / kScoreChunk;       // 0..3
  for (int c0 = 0; c0 < nT; c0 += kScoreChunk) {
    __syncthreads();
    const int ncol = min(kScoreChunk, nT - c0);
    for (int e = threadIdx.x; e < kScoreChunk * (D / 4); e += kScoreThreads) {
      const int cc = e / (D / 4), k4 = e % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (cc < ncol) v = *reinterpret_cast<const float4*>(kp + static_cast<size_t>(c0 + cc) * D + 4 * k4);
      kT[(4 * k4 + 0) * kKtStride + cc] = v.x;
      kT[(4 * k4 + 1) * kKtStride + cc] = v.y;
      kT[(4 * k4 + 2) * kKtStride + cc] = v.z;
      kT[(4 * k4 + 3) * kKtStride + cc] = v.w;
    }
    __syncthreads();
    float acc[RPT];
#pragma unroll
    for (int e = 0; e < RPT; ++e) acc[e] = 0.f;
    const float* q0 = qb + (rg * RPT) * D;
#pragma unroll 8
    for (int kk = 0; kk < D; ++kk) {
      const float kv = kT[kk * kKtStride + jj];
#pragma unroll
      for (int e = 0; e < RPT; ++e) acc[e] = fmaf(q0[e * D + kk], kv, acc[e]);
    }
    if (jj < ncol) {
      uint32_t* kr = keys + (rg * RPT) * nT + c0 + jj;
#pragma unroll
      for (int e = 0; e < RPT; ++e) kr[e * nT] = order_key(acc[e] + 0.f);
    }
  }
  __syncthreads();

  // top-k phase: warp w handles rows w, w + 8, ...
  const int warp = threadIdx.x / 32;
  for (int r = warp; r < nrows; r += kScoreThreads / 32)
    radix_topk_row(keys + r * nT, nT, topk, hist_all + warp * 256,
                   idx + (static_cast<size_t>(bh) * nT + row0 + r) * topk);
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads) score_topk_small_kernel(Geom g, const float* __restrict__ pooled,
                                                                         int topk, int32_t* __restrict__ idx) {
  constexpr int R = 8;
  constexpr int C4 = D / 4;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int nT = g.nT;
  float4* qb = reinterpret_cast<float4*>(smem_raw);
  float4* kb = qb + R * C4;
  uint32_t* keys = reinterpret_cast<uint32_t*>(kb + nT * C4);
  uint32_t* hist_all = keys + R * nT;

  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * R;
  const int nrows = min(R, nT - row0);
  const size_t BH = static_cast<size_t>(g.B) * g.H;
  const float4* qp = reinterpret_cast<const float4*>(pooled + (static_cast<size_t>(bh) * nT + row0) * D);
  const float4* kp = reinterpret_cast<const float4*>(pooled + ((BH + bh) * nT) * D);
  for (int e = threadIdx.x; e < R * C4; e += kScoreThreads)
    qb[e] = (e / C4 < nrows) ? qp[e] : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int e = threadIdx.x; e < nT * C4; e += kScoreThreads) kb[e] = kp[e];
  __syncthreads();

  const int lane = threadIdx.x % 32;
  for (int j = threadIdx.x; j < nT; j += kScoreThreads) {
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    const float4* krow = kb + j * C4;
#pragma unroll 4
    for (int i = 0; i < C4; ++i) {
      const int c = (i + lane) % C4;
      const float4 kv = krow[c];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 qv = qb[r * C4 + c];
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) keys[r * nT + j] = order_key(acc[r] + 0.f);
  }
  __syncthreads();

  const int warp = threadIdx.x / 32;
  if (warp < nrows)
    radix_topk_row(keys + warp * nT, nT, topk, hist_all + warp * 256,
                   idx + (static_cast<size_t>(bh) * nT + row0 + warp) * topk);
}

}  // namespace vsa
