// select_kernels.cuh -- tile selection: mean-pooling, tile scores, top-k.
//
// FastVideo VSA user guide (intro): for every query block, VSA scores the
// key/value blocks and keeps the top-k ("Wan top-k behavior": top-k counts
// key/value blocks per query block).  Scores are dot products of the tiles'
// mean-pooled Q and K.  fastbsa page ("How it works"): selection stays in
// shared memory instead of round-tripping a score matrix through HBM.
//
// Two kernels:
//   pool_kernel        HBM-bound: reads every Q and K byte once and writes the
//                      per-tile float32 means, channel-major, to the caller's
//                      workspace: Q means [B*H, d, ldq], then K means
//                      [B*H, d, ldk] (ldq, ldk: nTq, nTk rounded up to 4).
//   score_topk_kernel  per (head, block of R query tiles): the R x nTk score
//                      rows in shared memory (float32 FMA, channels summed in
//                      ascending order) and each row's exact top-k; writes
//                      ascending idx.  Launched as a programmatic dependent of
//                      the pooling grid, so its launch overlaps the pooling
//                      tail; it waits for the pooled means before reading them.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include <cuda.h>

#include "vsa_geometry.cuh"
#include "vsa_ptx.cuh"

namespace vsa {

constexpr int kPoolThreads = 256;

// Row stride (floats) of the transposed tile means.
__host__ __device__ inline int means_ld(int nT) { return (nT + 3) & ~3; }

inline size_t select_workspace_bytes(const Geom& gq, const Geom& gk) {
  return sizeof(float) * static_cast<size_t>(gq.B) * gq.H * gq.d * (means_ld(gq.nT) + means_ld(gk.nT));
}

// The coarse branch also pools V (its means follow the K means).
inline size_t coarse_workspace_bytes(const Geom& gq, const Geom& gk) {
  return sizeof(float) * static_cast<size_t>(gq.B) * gq.H * gq.d * (means_ld(gq.nT) + 2 * means_ld(gk.nT));
}

// Start of head bh's means of tensor z (0: Q, 1: K, 2: V) in the workspace.
__host__ __device__ inline size_t means_offset(const Geom& gq, const Geom& gk, int z, int bh) {
  const size_t BH = static_cast<size_t>(gq.B) * gq.H;
  const size_t kv = static_cast<size_t>(gk.d) * means_ld(gk.nT);
  return z == 0 ? static_cast<size_t>(bh) * gq.d * means_ld(gq.nT)
                : BH * gq.d * means_ld(gq.nT) + (z == 2 ? BH * kv : 0) + static_cast<size_t>(bh) * kv;
}

// Larger float -> larger unsigned key (total order; -0 < +0, scores are
// canonicalised so -0 does not occur).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Order key of an always-kept (prefix) tile: above every finite score's key.
constexpr uint32_t kKeepKey = 0xffffffffu;

// Exact top-k of one row of order keys by one warp, keys held in registers
// (lane l holds tiles l, l + 32, ...).  The topk-th largest key T is found
// from the top bit down.  Bits on which all keys agree are decided without
// counting.  With a scratch histogram (256 words of shared memory for the
// warp), 8 bits at a time are decided by a pass over the candidates (the
// keys sharing T's decided bits, at first all): each adds one to the bin of
// its next 8-bit digit (shared-memory atomics), a warp scan of the bins from
// the top finds the digit d of the topk-th key and adds the candidates of
// higher bins to `above`; d's bin holds the next candidates.  Passes repeat
// (at most three) while more than 128 candidates remain; when d's bin holds
// exactly the keys still missing, T is decided, else the candidates (at most
// 128, else all keys) are gathered into four registers per lane and the
// remaining bits are decided one by one on them: T keeps a bit when at least
// topk keys are >= T with that bit set (above + a warp-wide count over the
// gathered keys).  The
// search stops once exactly topk keys are >= T.  Every key above T is taken,
// then the keys equal to T in ascending tile order until topk are taken (ties
// go to the lower tile index); indices are written in ascending order.  Order
// keys of finite scores are never 0, so 0 marks padding slots.
template <int MAXE>
__device__ __forceinline__ void bsearch_topk_row(const uint32_t* kr, int nT, int topk, int32_t* out,
                                                 uint32_t* hist = nullptr) {
  const int lane = threadIdx.x % 32;
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t key[MAXE];
  uint32_t kand = 0xffffffffu, kor = 0u;
#pragma unroll
  for (int e = 0; e < MAXE; ++e) {
    const int j = lane + 32 * e;
    key[e] = (j < nT) ? kr[j] : 0u;
    if (j < nT) {
      kand &= key[e];
      kor |= key[e];
    }
  }
  kand = __reduce_and_sync(0xffffffffu, kand);
  kor = __reduce_or_sync(0xffffffffu, kor);
  const int common = __clz(kand ^ kor);          // leading bits shared by all keys (32: all equal)
  uint32_t T = common == 0 ? 0u : (kand & (0xffffffffu << (32 - common)));
  int b_next = 31 - common;                      // highest undecided bit
  bool gathered = false, done = false;
  uint32_t above = 0u;                           // keys above the candidates (the bins passed over)
  uint32_t g[4] = {0u, 0u, 0u, 0u};             // the gathered candidates, lane l: l, l + 32, ...
  if (hist != nullptr) {
    uint32_t ncand = static_cast<uint32_t>(nT); // keys sharing T's decided bits
    for (int pass = 0; pass < 3 && !done && b_next >= 7 && ncand > 128u; ++pass) {
      const int sh = b_next - 7;                 // digit = bits b_next .. sh
      const uint32_t hi = b_next == 31 ? 0u : (0xffffffffu << (b_next + 1));   // decided bits
      for (int i = lane; i < 256; i += 32) hist[i] = 0u;
      __syncwarp();
#pragma unroll
      for (int e = 0; e < MAXE; ++e)
        if (lane + 32 * e < nT && (key[e] & hi) == (T & hi)) atomicAdd(hist + ((key[e] >> sh) & 255u), 1u);
      __syncwarp();
      // lane l holds bins 255 - 8l .. 248 - 8l; candidates in higher bins by a scan
      const uint4 ha = *reinterpret_cast<const uint4*>(hist + 248 - 8 * lane);
      const uint4 hb = *reinterpret_cast<const uint4*>(hist + 252 - 8 * lane);
      const uint32_t h[8] = {hb.w, hb.z, hb.y, hb.x, ha.w, ha.z, ha.y, ha.x};   // bins 255-8l downwards
      uint32_t own = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) own += h[i];
      uint32_t incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t need = static_cast<uint32_t>(topk) - above;
      uint32_t run = incl - own;                 // candidates in bins above this lane's
      int dig = -1;
      uint32_t abv = 0u, cnt_d = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (dig < 0 && run + h[i] >= need) {
          dig = 255 - 8 * lane - i;
          abv = run;
          cnt_d = h[i];
        }
        run += h[i];
      }
      const uint32_t who = __ballot_sync(0xffffffffu, dig >= 0);
      const int src = __ffs(who) - 1;            // the lowest lane holds the highest qualifying bin
      dig = __shfl_sync(0xffffffffu, dig, src);
      above += __shfl_sync(0xffffffffu, abv, src);
      ncand = __shfl_sync(0xffffffffu, cnt_d, src);
      T |= static_cast<uint32_t>(dig) << sh;
      b_next = sh - 1;
      // every candidate of bin d is in: T (low bits 0) decides
      if (above + ncand == static_cast<uint32_t>(topk)) done = true;
      __syncwarp();                              // every lane has read the bins
    }
    if (!done && ncand <= 128u) {
      // gather the candidates (keys sharing T's decided bits) into registers
      const uint32_t hi = b_next >= 31 ? 0u : (0xffffffffu << (b_next + 1));
      const uint32_t lt_m = (1u << lane) - 1u;
      uint32_t base = 0u;
#pragma unroll
      for (int e = 0; e < MAXE; ++e) {
        const bool in = lane + 32 * e < nT && (key[e] & hi) == (T & hi);
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        if (in) hist[base + __popc(m & lt_m)] = key[e];
        base += __popc(m);
      }
      __syncwarp();
#pragma unroll
      for (int m = 0; m < 4; ++m) g[m] = lane + 32 * m < static_cast<int>(ncand) ? hist[lane + 32 * m] : 0u;
      gathered = true;
    } else {
      above = 0u;                                // count over all keys below
    }
    __syncwarp();                                // the scratch is reused by the warp's next row
  }
  if (!done) {
    for (int b = b_next; b >= 0; --b) {
      const uint32_t cand = T | (1u << b);
      uint32_t c;
      if (gathered) {
        c = above + __reduce_add_sync(0xffffffffu, ((g[0] >= cand ? 1u : 0u) + (g[1] >= cand ? 1u : 0u)) +
                                                       ((g[2] >= cand ? 1u : 0u) + (g[3] >= cand ? 1u : 0u)));
      } else {
        uint32_t p[4] = {0u, 0u, 0u, 0u};        // four independent chains of adds
#pragma unroll
        for (int e = 0; e < MAXE; ++e) p[e & 3] += (key[e] >= cand) ? 1u : 0u;
        c = __reduce_add_sync(0xffffffffu, (p[0] + p[1]) + (p[2] + p[3]));
      }
      if (c >= static_cast<uint32_t>(topk)) {
        T = cand;
        // exactly topk keys are >= T: they are the answer whatever the lower bits
        if (c == static_cast<uint32_t>(topk)) break;
      }
    }
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

// One CTA per (tile j, head bh, tensor z in {Q, K} -- and V for the coarse
// branch), each side with its own grid and tile (CTAs past a side's tile
// count exit).  The whole tile is one
// 5-D TMA box per 64-channel slab (the same views the attend kernel uses), so
// a 256-token tile of d = 128 puts 64 KB in flight per CTA without using
// registers; positions past the y and x edges arrive as zeros, and rows past
// the t edge are left out of the sums (in the [B, N, H, d] view they hold the
// next batch's frames).  Threads sum 16-byte chunks down the rows in a fixed
// order (deterministic) and divide by the tile's valid count.
// Dynamic shared memory: box (slabs x vol x 128 B, 1024-aligned) | partial sums | mbarrier.
template <int D, bool F16>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                            const __grid_constant__ CUtensorMap tmK,
                                                            const __grid_constant__ CUtensorMap tmV, Geom gq,
                                                            Geom gk, float* __restrict__ means, unsigned int* err) {
  constexpr int kSlabs = D / 64;
  constexpr int TPR = D / 8;                 // threads per row (one 16-byte chunk each)
  constexpr int RP = kPoolThreads / TPR;     // row groups
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sp = smem_raw + (base - raw);
  const int z = blockIdx.z;
  const Geom& g = z == 0 ? gq : gk;
  const int j = blockIdx.x;
  if (j >= g.nT) return;
  const int vol = g.vol;
  const int box_bytes = vol * 128;
  float* part = reinterpret_cast<float*>(sp + kSlabs * box_bytes);     // [RP][D]
  const uint32_t bar = base + kSlabs * box_bytes + RP * D * 4;

  const int bh = blockIdx.y;
  const TileCoord c = tile_coord(g, j);
  int vt, vy, vx;
  tile_extent(g, c, vt, vy, vx);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kSlabs * box_bytes));
    const BoxCoord bc = box_coord(g, bh, c.bt * g.tt, c.by * g.th, c.bx * g.tw);
    for (int sl = 0; sl < kSlabs; ++sl)
      tma_load_5d(base + sl * box_bytes,
                  z == 0 ? static_cast<const void*>(&tmQ)
                         : (z == 1 ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmV)),
                  bar, sl * 64, bc.c1, bc.c2, bc.c3, bc.c4);
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
  const int rows = vt * g.th * g.tw;          // rows of the box inside the t extent
  if (ok) {
#pragma unroll 4
    for (int r = rg; r < rows; r += RP) {
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
  const float cnt = static_cast<float>(vt * vy * vx);
  const int ld = means_ld(g.nT);
  float* mz = means + means_offset(gq, gk, z, bh);
  for (int col = threadIdx.x; col < D; col += kPoolThreads) {
    float sum = 0.f;
#pragma unroll 8
    for (int i = 0; i < RP; ++i) sum += part[i * D + col];
    mz[static_cast<size_t>(col) * ld + j] = sum / cnt;
  }
}

template <int D>
inline size_t pool_smem_bytes(const Geom& g) {
  return static_cast<size_t>(D / 64) * g.vol * 128 + (kPoolThreads / (D / 8)) * D * 4 + 16 + 1024;
}

// ------------------------------------------------------------ score + top-k
// Shared-memory traffic bounds the score phase: a 16-byte shared load is
// served one 8-lane quarter-warp at a time, so each costs at least four
// shared-memory cycles even when lanes read the same address.  A thread block
// of m x n scores per thread needs (m + n) such cycles per warp and channel
// for 32 m n FMAs, and the SM retires 128 FMAs per shared-memory cycle: the
// 8 x 8 block of the wide kernel balances the two (4 x 4 would run at half
// the FMA rate).

// One warp per row picks each row's top-k from the order keys in shared memory;
// `scratch` (16-byte aligned, 256 words per warp) holds each warp's histogram.
__device__ __forceinline__ void topk_rows(const uint32_t* keys, int kst, int nT, int nrows, int topk,
                                          int32_t* out_rows, int warps, uint32_t* scratch) {
  const int warp = threadIdx.x / 32;
  uint32_t* hist = scratch + 256 * warp;
  for (int r = warp; r < nrows; r += warps) {
    const uint32_t* kr = keys + r * kst;
    int32_t* out = out_rows + static_cast<size_t>(r) * topk;
    if (nT <= 32 * 8)
      bsearch_topk_row<8>(kr, nT, topk, out, hist);
    else if (nT <= 32 * 12)
      bsearch_topk_row<12>(kr, nT, topk, out, hist);
    else if (nT <= 32 * 16)
      bsearch_topk_row<16>(kr, nT, topk, out, hist);
    else if (nT <= 32 * 24)
      bsearch_topk_row<24>(kr, nT, topk, out, hist);
    else
      bsearch_topk_row<48>(kr, nT, topk, out, hist);
  }
}

// Wide kernel (heads of kNarrowMaxTiles + 1 .. kWideLongMaxTiles tiles): one CTA per (block of 32
// query tiles, head), 8 warps.  Per pass of 512 key tiles, warp w takes key
// tiles 64w .. 64w + 63 of the pass against all 32 query tiles; lane
// (qg = lane / 8, kg = lane % 8) holds the 8 x 8 block of query tiles
// {4qg .. 4qg+3, 16+4qg .. 16+4qg+3} x key tiles {4kg .. 4kg+3, 32+4kg ..
// 32+4kg+3} of the warp's 64, so each 16-byte load of a quarter-warp covers
// 128 contiguous bytes (no bank conflicts).  Key means stream through shared
// memory in slices of 16 channels x 512 key tiles on a cp.async ring, 3 deep
// (2 past kWideMaxTiles key tiles, where the key rows need the room)
// (one barrier per slice).  Warps whose key tiles lie past nT skip the math.
// Each score adds its channels in ascending order (deterministic); scores
// become order keys in shared memory, never written to HBM.
// Dynamic shared memory: qT [D][32] | ring [STAGES][16][512] | keys [32][nT].
constexpr int kWideRows = 32;
constexpr int kWideKeys = 512;        // key tiles per pass (8 math warps), heads of up to 512
constexpr int kWideKeysOne = 768;     // one pass of 768 (12 math warps) for 513-768 key tiles
constexpr int kWideSlice = 16;
constexpr int kWideStages = 3;        // ring depth up to kWideMaxTiles key tiles
constexpr int kWideStagesLong = 2;    // ring depth up to kWideLongMaxTiles (room for the key rows)
constexpr int kWideThreads = 512;     // warps past KEYS / 64 help only with copies and the top-k
constexpr int kWideMaxTiles = 768;
constexpr int kWideLongMaxTiles = 1024;
constexpr int kNarrowMaxTiles = 256;   // below this the narrow kernel is used too (more, shorter CTAs)

template <int D, int STAGES, int KEYS>
__global__ void __launch_bounds__(kWideThreads, 1) score_topk_kernel(Geom gq, Geom gk, const float* __restrict__ means, int topk,
                                                                  int32_t* __restrict__ idx) {
  constexpr int SPP = D / kWideSlice;      // stages per pass
  constexpr int SLICE = kWideSlice * KEYS;
  constexpr int MW = KEYS / 64;            // math warps: 64 key tiles each
  constexpr int R = kWideRows;
  // the pooled means are written by the previous grid: wait for it
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qT = reinterpret_cast<float*>(smem_raw);
  float* ring = qT + D * R;
  uint32_t* keys = reinterpret_cast<uint32_t*>(ring + STAGES * SLICE);
  const int nT = gk.nT;                     // key tiles (score columns, top-k candidates)
  const int ldq = means_ld(gq.nT), ldk = means_ld(nT);
  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * R;
  const int nrows = min(R, gq.nT - row0);
  const float* mq = means + means_offset(gq, gk, 0, bh);
  const float* mk = means + means_offset(gq, gk, 1, bh);
  const int nstage = ceil_div(nT, KEYS) * SPP;

  // query means (joined to the first cp.async group); float4s past the row are zero
  for (int f = threadIdx.x; f < D * R / 4; f += kWideThreads) {
    const int c = f / (R / 4), r4 = f % (R / 4);
    const int row = row0 + 4 * r4;
    const bool in = row < ldq;
    cp_async16(smem_u32(qT + c * R + 4 * r4),
               in ? static_cast<const void*>(mq + static_cast<size_t>(c) * ldq + row) : static_cast<const void*>(mq),
               in ? 16u : 0u);
  }
  // stage st = (pass st / SPP, channel slice st % SPP) -> ring slot st % 3; one group per call
  auto issue = [&](int st) {
    if (st < nstage) {
      const int kc0 = (st / SPP) * KEYS, c0 = (st % SPP) * kWideSlice;
      float* dst = ring + (st % STAGES) * SLICE;
#pragma unroll 4
      for (int f = threadIdx.x; f < SLICE / 4; f += kWideThreads) {
        const int c = f / (KEYS / 4), k4 = f % (KEYS / 4);
        const int key = kc0 + 4 * k4;
        const bool in = key < ldk;
        cp_async16(smem_u32(dst + c * KEYS + 4 * k4),
                   in ? static_cast<const void*>(mk + static_cast<size_t>(c0 + c) * ldk + key)
                      : static_cast<const void*>(mk),
                   in ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int st = 0; st < STAGES - 1; ++st) issue(st);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qg = lane / 8, kg = lane % 8;
  // acc2[i][p] holds the scores of query tile i with key tiles 2p, 2p + 1 of
  // the block: packed fma.rn.f32x2, each lane the same fused multiply-add in
  // the same channel order as a scalar one
  uint64_t acc2[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int p = 0; p < 4; ++p) acc2[i][p] = 0ull;

  for (int st = 0; st < nstage; ++st) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();                 // slice st visible; slot of slice st-1 free
    issue(st + STAGES - 1);
    const int sl = st % SPP;
    const int kw0 = (st / SPP) * KEYS + 64 * warp;   // the warp's first key tile
    if (warp < MW && kw0 < nT) {
      const float* kb = ring + (st % STAGES) * SLICE + 64 * warp + 4 * kg;
      const float* qb = qT + sl * kWideSlice * R + 4 * qg;
#pragma unroll
      for (int c = 0; c < kWideSlice; ++c) {
        const float4 q0 = *reinterpret_cast<const float4*>(qb + c * R);
        const float4 q1 = *reinterpret_cast<const float4*>(qb + c * R + 16);
        const float4 k0 = *reinterpret_cast<const float4*>(kb + c * KEYS);
        const float4 k1 = *reinterpret_cast<const float4*>(kb + c * KEYS + 32);
        const float qa[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        const uint64_t kp[4] = {f2_pack(k0.x, k0.y), f2_pack(k0.z, k0.w), f2_pack(k1.x, k1.y), f2_pack(k1.z, k1.w)};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint64_t qq = f2_pack(qa[i], qa[i]);
#pragma unroll
          for (int p = 0; p < 4; ++p) acc2[i][p] = f2_fma(qq, kp[p], acc2[i][p]);
        }
      }
    }
    if (sl == SPP - 1 && warp < MW) {   // end of a pass: scores -> order keys
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = (i < 4 ? 0 : 16) + 4 * qg + (i & 3);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float sc[2];
          f2_unpack(acc2[i][p], sc[0], sc[1]);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 2 * p + h;
            const int key = kw0 + (j < 4 ? 0 : 32) + 4 * kg + (j & 3);
            if (row < nrows && key < nT) keys[row * nT + key] = key < gk.prefix ? kKeepKey : order_key(sc[h] + 0.f);
          }
          acc2[i][p] = 0ull;
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  // (the ring is free now: it holds the warps' histograms)
  topk_rows(keys, nT, nT, nrows, topk, idx + (static_cast<size_t>(bh) * gq.nT + row0) * topk, kWideThreads / 32,
            reinterpret_cast<uint32_t*>(ring));
}

template <int D, int STAGES, int KEYS>
inline size_t score_smem_bytes(const Geom& gk) {
  return sizeof(float) * (static_cast<size_t>(D) * kWideRows + STAGES * kWideSlice * KEYS) +
         sizeof(uint32_t) * static_cast<size_t>(kWideRows) * gk.nT;
}

// Narrow kernel (heads of at most kNarrowMaxTiles tiles, and of more than
// kWideLongMaxTiles, whose 32 key rows would not fit beside the wide ring): one
// CTA per (block of 16 query tiles, head), 8 warps; lane (qg, kg) of warp w
// holds the 4 x 4 block of query tiles 4qg .. 4qg+3 x key tiles 32w + 4kg ..
// 32w + 4kg + 3 of a pass of KEYS key tiles (KEYS / 32 warps do the math).
// Key means stream in slices of 16 channels x KEYS key tiles on a STAGES-deep
// cp.async ring: 256-key passes on a 4-deep ring, or, for heads of at most
// 128 tiles, 128-key passes on an 8-deep ring, so every slice of the single
// pass is in flight at once (one L2 round trip instead of one per slice).
// Same summation order and selection as the wide kernel.
// Dynamic shared memory: qT [D][16] | ring [STAGES][16][KEYS] | keys [16][nT].
constexpr int kNarrowRows = 16;
constexpr int kNarrowKeys = 256;
constexpr int kNarrowSlice = 16;
constexpr int kNarrowStages = 4;
constexpr int kShortKeys = 128;       // heads of at most kShortKeys tiles
constexpr int kShortStages = 8;
constexpr int kNarrowThreads = 256;   // two CTAs per SM at small tile counts

template <int D, int KEYS, int STAGES>
__global__ void __launch_bounds__(kNarrowThreads) score_topk_narrow_kernel(Geom gq, Geom gk, const float* __restrict__ means,
                                                                           int topk, int32_t* __restrict__ idx) {
  constexpr int SPP = D / kNarrowSlice;
  constexpr int SLICE = kNarrowSlice * KEYS;
  constexpr int MW = KEYS / 32;             // math warps
  constexpr int R = kNarrowRows;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qT = reinterpret_cast<float*>(smem_raw);
  float* ring = qT + D * R;
  uint32_t* keys = reinterpret_cast<uint32_t*>(ring + STAGES * SLICE);
  const int nT = gk.nT;                     // key tiles (score columns, top-k candidates)
  const int ldq = means_ld(gq.nT), ldk = means_ld(nT);
  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * R;
  const int nrows = min(R, gq.nT - row0);
  const float* mq = means + means_offset(gq, gk, 0, bh);
  const float* mk = means + means_offset(gq, gk, 1, bh);
  const int nstage = ceil_div(nT, KEYS) * SPP;

  for (int f = threadIdx.x; f < D * R / 4; f += kNarrowThreads) {
    const int c = f / (R / 4), r4 = f % (R / 4);
    const int row = row0 + 4 * r4;
    const bool in = row < ldq;
    cp_async16(smem_u32(qT + c * R + 4 * r4),
               in ? static_cast<const void*>(mq + static_cast<size_t>(c) * ldq + row) : static_cast<const void*>(mq),
               in ? 16u : 0u);
  }
  auto issue = [&](int st) {
    if (st < nstage) {
      const int kc0 = (st / SPP) * KEYS, c0 = (st % SPP) * kNarrowSlice;
      float* dst = ring + (st % STAGES) * SLICE;
      for (int f = threadIdx.x; f < SLICE / 4; f += kNarrowThreads) {
        const int c = f / (KEYS / 4), k4 = f % (KEYS / 4);
        const int key = kc0 + 4 * k4;
        const bool in = key < ldk;
        cp_async16(smem_u32(dst + c * KEYS + 4 * k4),
                   in ? static_cast<const void*>(mk + static_cast<size_t>(c0 + c) * ldk + key)
                      : static_cast<const void*>(mk),
                   in ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int st = 0; st < STAGES - 1; ++st) issue(st);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qg = lane / 8, kg = lane % 8;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int st = 0; st < nstage; ++st) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    issue(st + STAGES - 1);
    const int sl = st % SPP;
    const float* kb = ring + (st % STAGES) * SLICE + 32 * (warp % MW) + 4 * kg;
    const float* qb = qT + sl * kNarrowSlice * R + 4 * qg;
    if (warp < MW) {
#pragma unroll
      for (int c = 0; c < kNarrowSlice; ++c) {
        const float4 qv = *reinterpret_cast<const float4*>(qb + c * R);
        const float4 kv = *reinterpret_cast<const float4*>(kb + c * KEYS);
        const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
        const float ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qa[i], ka[j], acc[i][j]);
      }
    }
    if (sl == SPP - 1 && warp < MW) {
      const int kc0 = (st / SPP) * KEYS + 32 * warp + 4 * kg;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (4 * qg + i < nrows && kc0 + j < nT)
            keys[(4 * qg + i) * nT + kc0 + j] = kc0 + j < gk.prefix ? kKeepKey : order_key(acc[i][j] + 0.f);
          acc[i][j] = 0.f;
        }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  topk_rows(keys, nT, nT, nrows, topk, idx + (static_cast<size_t>(bh) * gq.nT + row0) * topk, kNarrowThreads / 32,
            reinterpret_cast<uint32_t*>(ring));
}

template <int D, int KEYS, int STAGES>
inline size_t score_narrow_smem_bytes(const Geom& gk) {
  return sizeof(float) * (static_cast<size_t>(D) * kNarrowRows + STAGES * kNarrowSlice * KEYS) +
         sizeof(uint32_t) * static_cast<size_t>(kNarrowRows) * gk.nT;
}

// ------------------------------------------------------------ coarse branch
// Tile-level attention (pooled coarse branch): for query tile i of head bh,
// o[i] = sum_j softmax_j(scale * qbar_i . kbar_j) vbar_j over every
// key/value tile j, from the channel-major means in the workspace.  One CTA
// per (8 * QT query tiles, head); each warp takes QT query tiles and lane l
// holds their scores for key tiles l, l + 32, ... (QT tiles per warp, so
// each mean read from shared memory feeds QT FMAs: with one, the kernel ran
// at the shared-memory bandwidth).  The key means, then the value means,
// stream through shared memory in slices of kCoarseSlice channels on a
// cp.async ring (kCoarseStages deep, one barrier per slice), each slice read
// from L2 once per CTA.  The softmax is a warp reduction between the two
// passes, and each output channel a warp sum of p_j * vbar_j[c].  float32
// throughout.
constexpr int kCoarseWarps = 8;
constexpr int kCoarseSlice = 8;
constexpr int kCoarseStages = 3;

template <int D, int MAXJ, int QT>
__global__ void __launch_bounds__(kCoarseWarps * 32) coarse_kernel(Geom gq, Geom gk, const float* __restrict__ means,
                                                                   float scale_log2, float* __restrict__ out) {
  constexpr int SPP = D / kCoarseSlice;            // slices per pass
  extern __shared__ __align__(16) float csm[];
  float* qs = csm;                                  // [kCoarseWarps * QT][D]
  float* ring = csm + kCoarseWarps * QT * D;        // [kCoarseStages][kCoarseSlice][ldk]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  const int i0 = (blockIdx.x * kCoarseWarps + warp) * QT;       // the warp's first query tile
  const int nT = gk.nT, ldq = means_ld(gq.nT), ldk = means_ld(nT);
  const float* mq = means + means_offset(gq, gk, 0, bh);
  const float* mk = means + means_offset(gq, gk, 1, bh);
  const float* mv = means + means_offset(gq, gk, 2, bh);
  const int slice_f = kCoarseSlice * ldk;           // floats per slice
  // slice st: K channels for st < SPP, then V channels; one cp.async group per call
  auto issue = [&](int st) {
    if (st < 2 * SPP) {
      const float* m = st < SPP ? mk : mv;
      const int c0 = (st % SPP) * kCoarseSlice;
      float* dst = ring + (st % kCoarseStages) * slice_f;
      for (int f = threadIdx.x; f < slice_f / 4; f += kCoarseWarps * 32) {
        const int c = (4 * f) / ldk, j = (4 * f) % ldk;
        cp_async16(smem_u32(dst + 4 * f), m + static_cast<size_t>(c0 + c) * ldk + j, 16u);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int st = 0; st < kCoarseStages - 1; ++st) issue(st);
  float* qw = qs + warp * QT * D;
#pragma unroll
  for (int u = 0; u < QT; ++u)
    for (int c = lane; c < D; c += 32) qw[u * D + c] = i0 + u < gq.nT ? mq[static_cast<size_t>(c) * ldq + i0 + u] : 0.f;
  float s[QT][MAXJ];
#pragma unroll
  for (int u = 0; u < QT; ++u)
#pragma unroll
    for (int t = 0; t < MAXJ; ++t) s[u][t] = 0.f;
  float inv_l[QT];
  for (int st = 0; st < 2 * SPP; ++st) {
    cp_async_wait<kCoarseStages - 2>();
    __syncthreads();                                // slice st visible; the slot of slice st-1 is free
    issue(st + kCoarseStages - 1);
    const float* sl = ring + (st % kCoarseStages) * slice_f;
    const int c0 = (st % SPP) * kCoarseSlice;
    if (st < SPP) {
#pragma unroll
      for (int c = 0; c < kCoarseSlice; ++c) {
        float qc[QT];
#pragma unroll
        for (int u = 0; u < QT; ++u) qc[u] = qw[u * D + c0 + c];
#pragma unroll
        for (int t = 0; t < MAXJ; ++t) {
          const int j = lane + 32 * t;
          if (j < nT) {
            const float kv = sl[c * ldk + j];
#pragma unroll
            for (int u = 0; u < QT; ++u) s[u][t] = fmaf(qc[u], kv, s[u][t]);
          }
        }
      }
      if (st == SPP - 1) {                          // scores complete: softmax weights
#pragma unroll
        for (int u = 0; u < QT; ++u) {
          float mx = -INFINITY;
#pragma unroll
          for (int t = 0; t < MAXJ; ++t) {
            s[u][t] = (lane + 32 * t < nT) ? s[u][t] * scale_log2 : -INFINITY;
            mx = fmaxf(mx, s[u][t]);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          float l = 0.f;
#pragma unroll
          for (int t = 0; t < MAXJ; ++t) {
            s[u][t] = ex2_approx(s[u][t] - mx);     // 0 past the last key tile
            l += s[u][t];
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
          inv_l[u] = 1.f / l;
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < kCoarseSlice; ++c) {
        float acc[QT];
#pragma unroll
        for (int u = 0; u < QT; ++u) acc[u] = 0.f;
#pragma unroll
        for (int t = 0; t < MAXJ; ++t) {
          const int j = lane + 32 * t;
          if (j < nT) {
            const float vv = sl[c * ldk + j];
#pragma unroll
            for (int u = 0; u < QT; ++u) acc[u] = fmaf(s[u][t], vv, acc[u]);
          }
        }
#pragma unroll
        for (int u = 0; u < QT; ++u) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
          if (i0 + u < gq.nT && lane == ((c0 + c) & 31))
            out[(static_cast<size_t>(bh) * gq.nT + i0 + u) * D + c0 + c] = acc[u] * inv_l[u];
        }
      }
    }
  }
  cp_async_wait<0>();
}

// Key tiles per lane (MAXJ) and query tiles per warp (QT) by key tile count.
template <int D>
inline size_t coarse_smem_bytes(const Geom& gk, int qt) {
  return sizeof(float) * (static_cast<size_t>(kCoarseWarps) * qt * D +
                          static_cast<size_t>(kCoarseStages) * kCoarseSlice * means_ld(gk.nT));
}

}  // namespace vsa
