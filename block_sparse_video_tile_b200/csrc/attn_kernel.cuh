// attn_kernel.cuh -- block-sparse flash-attention forward for sm_100a.
//
// FastVideo VSA user guide (intro): each query block attends only to the
// tokens of its selected top-k key/value blocks; "Verify routing and
// fallback": non-causal self-attention, scale head_size ** -0.5 by default.
// fastbsa page ("How it works"): Q/K/V stay in raster layout and the block
// index map is evaluated in the kernel (here: 5-D TMA boxes over
// [B*H, T, Hh, W, d], so a tile or half-tile is one box, zero-filled past the
// grid edge).
//
// One CTA = one work unit with two "slots" of 128 query rows each.
//   MODE_SHARED (tiles of 256 tokens, tt >= 2): the slots are the two t-halves
//     of one query tile and share every K/V sub-block (a t-half of a kept tile).
//   MODE_TILE (tiles of 128 tokens): each slot is one query tile; a K/V
//     sub-block is one of its kept tiles.
//   MODE_PAIR (tiles of 64 tokens): each slot stacks two neighbouring query
//     tiles A (rows 0-63) and B (rows 64-127).  The slot walks the union of
//     their kept lists, two 64-token tiles per K/V sub-block, and every row
//     masks the tiles only the other query tile kept.  Neighbouring tiles of a
//     video keep mostly the same tiles, so most of each 128-row MMA is useful
//     work; at worst (disjoint lists) it is half, as with one padded tile.
// Warp roles (384 threads): warps 0-3 softmax slot 0, warps 4-7 softmax slot 1
// (thread = query row = TMEM lane); warp 9 + h issues slot h's MMAs; warp 8
// is the TMA producer (for both slots in MODE_SHARED, whose slots share one
// K/V stream; for slot 0 otherwise, with warp 11 producing slot 1), and in
// MODE_PAIR warps 10-11 first build the union lists.  The producer warpgroup
// gives registers to the softmax warpgroups (setmaxnreg, RegSplit: 208/88, or
// 200/96 in MODE_PAIR, within the launch's 384*168).
// TMEM (512 columns): S_h at [128h, 128h+128), P_h (16-bit pairs) aliases the
// first 64 columns of S_h, O_h at [256 + 128h, ...).  Per K/V sub-block the
// MMA groups enter the tensor pipe in the order PV_0(prev), S_0(cur),
// PV_1(prev), S_1(cur) (the two issuers pass a token); one thread issues a
// slot's MMAs, and tcgen05.mma ops from one thread execute in issue order, so
// S_h(cur) overwrites P_h(prev) only after PV_h(prev) has read it, and
// softmax h works while the tensor pipe runs the other slot.  Online softmax in float32 with lazy rescaling (O
// and l are only rescaled when the running max grows by more than 2^8).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "vsa_geometry.cuh"
#include "vsa_ptx.cuh"

namespace vsa {

constexpr int kAttnThreads = 384;        // 3 warpgroups
// Registers per thread after setmaxnreg: warpgroups 0-1 (softmax) and 2 (TMA
// and MMA warps).  2*128*S + 128*P must stay within the launch's 384*168.
// In MODE_PAIR the producer and issuer warps walk union lists (pieces with
// membership flags) and the softmax has less to hold, so 8 registers move to
// the producer warpgroup (fewer spills and faster, measured).
template <int MODE>
struct RegSplit {
  static constexpr int kSoftmax = MODE == 2 ? 200 : 208;
  static constexpr int kProducer = MODE == 2 ? 96 : 88;
  static_assert(2 * 128 * kSoftmax + 128 * kProducer <= 384 * 168, "register split over the launch budget");
};
constexpr int kSlotRows = 128;          // MMA M
constexpr int kSubRows = 128;           // K/V rows per sub-block (S: N, PV: K)
constexpr float kRescaleLog2 = 8.0f;
#ifndef VSA_EXP_POLY_PER8
#define VSA_EXP_POLY_PER8 0
#endif
// Of every 8 column pairs of a score row, this many take 2^x on the FMA pipe
// (exp2_poly_pair) and the rest on the multi-function unit (ex2.approx): the
// two units then share the softmax's exponentials.
constexpr int kExpPolyPer8 = VSA_EXP_POLY_PER8;
#ifndef VSA_P_PACK_ALU
#define VSA_P_PACK_ALU 0
#endif
// Convert P to bf16 on the integer ALU (pack_bf16x2_alu) rather than with the
// float conversion instruction.
constexpr bool kPackAlu = VSA_P_PACK_ALU != 0;
constexpr uint32_t kErrBadIndex = 2u;

enum : int { MODE_SHARED = 0, MODE_TILE = 1, MODE_PAIR = 2 };

struct AttnArgs {
  Geom gq, gk;               // query side, key/value side (same tile volume)
  int topk;
  float scale_log2;          // softmax_scale * log2(e)
  const int32_t* idx;        // [B*H, nTq, topk], entries in [0, nTk)
  uint16_t* o;               // Q's layout, bf16 or fp16 like the inputs
  float* lse;                // [B*H, Nq]
  unsigned int* err;         // device error word
  int box_tq, box_tk;        // t-extent of one TMA box per side (tt/2 in MODE_SHARED, else tt)
};

template <int D>
struct AttnSmem {
  static constexpr int kSlabBytes = 128 * 128;       // 128 rows x 64 bf16 (one 128B-swizzle slab)
  static constexpr int kSlabs = D / 64;
  static constexpr int kBufBytes = kSlabs * kSlabBytes;
  static constexpr int kQ = 0;                        // 2 slot buffers
  static constexpr int kK = 2 * kBufBytes;            // 2 buffers
  static constexpr int kV = 4 * kBufBytes;            // 2 buffers
  static constexpr int kBar = 6 * kBufBytes;
  static constexpr int kNumBars = 17;
  static constexpr int kMisc = kBar + kNumBars * 8;   // TMEM address, abort flag, union lengths
  static constexpr int kTiles = kMisc + 16;           // uint2 per tile: (bt, by | bx << 16)
  // then, in MODE_PAIR only: membership bitmaps (4 x ceil(nT/32) words) and
  // the two slots' union lists (2 x 2*topk entries of j | in_a << 16 | in_b << 17)
  __host__ __device__ static int bitmap_off(int nT) { return kTiles + ((8 * nT + 15) & ~15); }
  __host__ __device__ static int bitmap_words(int nT) { return (nT + 31) / 32; }
  __host__ __device__ static int union_off(int nT) { return bitmap_off(nT) + ((16 * bitmap_words(nT) + 15) & ~15); }
  __host__ __device__ static int total(int nT, int topk, bool pair) {
    return pair ? union_off(nT) + 2 * 2 * topk * 4 : kTiles + 8 * nT;
  }
  __host__ __device__ static int alloc(int nT, int topk, bool pair) { return total(nT, topk, pair) + 1024; }
};

enum : int {
  BAR_Q_FULL = 0, BAR_K_FULL = 2, BAR_K_EMPTY = 4, BAR_V_FULL = 6, BAR_V_EMPTY = 8,
  BAR_S_FULL = 10, BAR_P_FULL = 12, BAR_O_FULL = 14, BAR_DRAIN = 16
};

struct Slot {
  bool active;
  int bh, tile;          // head index (b*H + h) and query tile (tile A in MODE_PAIR)
  int t0, y0, x0;        // origin of the slot's (first) query box
  bool has_b;            // MODE_PAIR: tile B = tile + 1 exists
  int tb0, yb0, xb0;     // MODE_PAIR: origin of tile B
};

// The key/value side's geometry and box t-extent.  SAME: the key/value side
// uses the query grid and tile, known at compile time, so the kernel reads
// one set of parameters (fewer live registers in the softmax warps).
template <bool SAME>
__device__ __forceinline__ const Geom& kv_geom(const AttnArgs& a) {
  return SAME ? a.gq : a.gk;
}
template <bool SAME>
__device__ __forceinline__ int kv_box_t(const AttnArgs& a) {
  return SAME ? a.box_tq : a.box_tk;
}

template <bool SAME>
__device__ __forceinline__ int load_tile_index(const AttnArgs& a, const int32_t* row, int e,
                                               bool report) {
  int j = __ldg(row + e);
  if (j < 0 || j >= kv_geom<SAME>(a).nT) {
    if (report) atomicCAS(a.err, 0u, kErrBadIndex);
    j = 0;
  }
  return j;
}

// Tile coordinates from the per-CTA table built at kernel start (one shared
// memory load instead of integer divisions in every iteration).
__device__ __forceinline__ TileCoord table_coord(const uint2* tab, int j) {
  const uint2 e = tab[j];
  TileCoord c;
  c.bt = static_cast<int>(e.x);
  c.by = static_cast<int>(e.y & 0xffffu);
  c.bx = static_cast<int>(e.y >> 16);
  return c;
}

// One K/V piece of a sub-block: kept tile j, t offset of the box inside the
// tile, whether it is real (false: padding that repeats a real tile, fully
// masked), and which query tile of a MODE_PAIR slot kept it.
struct Piece {
  int j, toff;
  bool real, in_a, in_b;
};

// K/V sub-block sequence of one slot.
//   MODE_SHARED: for each kept tile (ascending), its t-halves that hold a token.
//   MODE_TILE:   each kept tile.
//   MODE_PAIR:   the ascending union of tile A's and tile B's kept lists (built
//                in shared memory at kernel start), two tiles per sub-block (a
//                short last sub-block is padded).
template <int MODE, bool SAME>
struct KvSeq {
  const int32_t* row;     // kept list of the slot's (first) query tile
  const uint32_t* uni;    // MODE_PAIR: the slot's union list in shared memory
  int ulen;               // MODE_PAIR: its length
  const uint2* tab;
  int pos, half;

  __device__ void init(const AttnArgs& a, const uint2* table, int bh, int tile, const uint32_t* union_list = nullptr,
                       int union_len = 0) {
    row = a.idx + (static_cast<size_t>(bh) * a.gq.nT + tile) * a.topk;
    uni = union_list;
    ulen = union_len;
    tab = table;
    pos = 0;
    half = 0;
  }
  __device__ bool second_half(const AttnArgs& a, int j) const {
    return static_cast<int>(tab[j].x) * kv_geom<SAME>(a).tt + kv_box_t<SAME>(a) < kv_geom<SAME>(a).T;
  }
  __device__ int count(const AttnArgs& a) const {
    if (MODE == MODE_TILE) return a.topk;
    if (MODE == MODE_PAIR) return (ulen + 1) / 2;
    int n = 0;
    for (int e = 0; e < a.topk; ++e) n += 1 + (second_half(a, load_tile_index<SAME>(a, row, e, false)) ? 1 : 0);
    return n;
  }
  // Piece p (0 or 1) of the current sub-block.
  __device__ Piece piece(const AttnArgs& a, int p, bool report) const {
    Piece pc;
    if (MODE == MODE_SHARED) {
      pc.j = load_tile_index<SAME>(a, row, pos, report);
      pc.toff = half * kv_box_t<SAME>(a);
      pc.real = pc.in_a = pc.in_b = true;
    } else if (MODE == MODE_TILE) {
      pc.j = load_tile_index<SAME>(a, row, pos, report);
      pc.toff = 0;
      pc.real = pc.in_a = pc.in_b = true;
    } else {
      const int e = 2 * pos + p;
      const bool real = e < ulen;
      const uint32_t u = uni[real ? e : 2 * pos];   // padding repeats a real piece, all masked
      pc.j = static_cast<int>(u & 0xffffu);
      pc.toff = 0;
      pc.real = real;
      pc.in_a = real && ((u >> 16) & 1u);
      pc.in_b = real && ((u >> 17) & 1u);
    }
    return pc;
  }
  __device__ void advance(const AttnArgs& a) {
    if (MODE == MODE_SHARED) {
      if (half == 0 && second_half(a, load_tile_index<SAME>(a, row, pos, false))) {
        half = 1;
      } else {
        half = 0;
        ++pos;
      }
    } else {
      ++pos;
    }
  }
};

// One warp builds a MODE_PAIR slot's union list: membership bitmaps of the two
// kept lists, then the set tiles in ascending order with per-list flags
// (prefix counts across the warp give each tile its position).  Returns the
// union length (valid in every lane).
template <bool SAME>
__device__ __forceinline__ int build_union(const AttnArgs& a, const int32_t* row_a, bool has_b, uint32_t* bm_a,
                                           uint32_t* bm_b, uint32_t* out) {
  const int lane = threadIdx.x % 32;
  const int nw = (kv_geom<SAME>(a).nT + 31) / 32;
  for (int w = lane; w < nw; w += 32) {
    bm_a[w] = 0u;
    bm_b[w] = 0u;
  }
  __syncwarp();
  for (int e = lane; e < a.topk; e += 32) {
    const int ja = load_tile_index<SAME>(a, row_a, e, true);
    atomicOr(bm_a + (ja >> 5), 1u << (ja & 31));
    if (has_b) {
      const int jb = load_tile_index<SAME>(a, row_a + a.topk, e, true);
      atomicOr(bm_b + (jb >> 5), 1u << (jb & 31));
    }
  }
  __syncwarp();
  int base = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t ua = (w < nw) ? bm_a[w] : 0u;
    const uint32_t ub = (w < nw) ? bm_b[w] : 0u;
    uint32_t u = ua | ub;
    const int cnt = __popc(u);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int pos = base + incl - cnt;
    while (u) {
      const int b = __ffs(u) - 1;
      u &= u - 1;
      out[pos++] = static_cast<uint32_t>(32 * w + b) | (((ua >> b) & 1u) << 16) | (((ub >> b) & 1u) << 17);
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  return base;
}

template <int D, int MODE, bool F16, bool SAME, bool BNHD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  constexpr bool SHARED = MODE == MODE_SHARED;
  constexpr bool PAIR = MODE == MODE_PAIR;
  constexpr int P = PAIR ? 2 : 1;                            // pieces per K/V sub-block
  using L = AttnSmem<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sp = smem_raw + (base - raw);
  const uint32_t sQ = base + L::kQ, sK = base + L::kK, sV = base + L::kV, sBar = base + L::kBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + L::kMisc + 4);
  uint2* tile_tab = reinterpret_cast<uint2*>(sp + L::kTiles);
  int* union_len = reinterpret_cast<int*>(sp + L::kMisc + 8);          // [2]
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(sp + L::bitmap_off(kv_geom<SAME>(a).nT));
  uint32_t* unions = reinterpret_cast<uint32_t*>(sp + L::union_off(kv_geom<SAME>(a).nT));
  auto bar = [&](int id) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(id); };

  const Geom& g = a.gq;                                     // query side
  const Geom& gk = kv_geom<SAME>(a);                        // key/value side
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int box_rows = SHARED ? kSubRows : g.vol;          // rows per TMA box (equal volumes)
  const uint32_t box_bytes = static_cast<uint32_t>(box_rows) * 128u;

  // ---- work unit -> slots
  Slot slot[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    int bh, tile, toff;
    bool act;
    bool has_b = false;
    if (SHARED) {
      bh = blockIdx.x / g.nT;
      tile = blockIdx.x % g.nT;
      toff = h * a.box_tq;
      act = true;
    } else if (MODE == MODE_TILE) {
      const long long gidx = 2ll * blockIdx.x + h;
      act = gidx < static_cast<long long>(g.B) * g.H * g.nT;
      bh = act ? static_cast<int>(gidx / g.nT) : 0;
      tile = act ? static_cast<int>(gidx % g.nT) : 0;
      toff = 0;
    } else {
      const int npair = (g.nT + 1) / 2;
      const long long gp = 2ll * blockIdx.x + h;
      act = gp < static_cast<long long>(g.B) * g.H * npair;
      bh = act ? static_cast<int>(gp / npair) : 0;
      tile = act ? 2 * static_cast<int>(gp % npair) : 0;
      has_b = act && tile + 1 < g.nT;
      toff = 0;
    }
    const TileCoord c = tile_coord(g, tile);
    slot[h].bh = bh;
    slot[h].tile = tile;
    slot[h].t0 = c.bt * g.tt + toff;
    slot[h].y0 = c.by * g.th;
    slot[h].x0 = c.bx * g.tw;
    slot[h].active = act && slot[h].t0 < g.T;
    slot[h].has_b = has_b;
    const TileCoord cb = tile_coord(g, has_b ? tile + 1 : tile);
    slot[h].tb0 = cb.bt * g.tt;
    slot[h].yb0 = cb.by * g.th;
    slot[h].xb0 = cb.bx * g.tw;
  }
  const int last_active = slot[1].active ? 1 : 0;

  // ---- setup: tile table, barriers, zero rows of a missing tile B, TMEM
  for (int j = threadIdx.x; j < gk.nT; j += kAttnThreads) {
    const TileCoord c = tile_coord(gk, j);
    tile_tab[j] = make_uint2(static_cast<uint32_t>(c.bt),
                             static_cast<uint32_t>(c.by) | (static_cast<uint32_t>(c.bx) << 16));
  }
  if (threadIdx.x == 0) {
    // MODE_SHARED: each active slot's issuer releases every K/V stage and drains
    const uint32_t n_issuers = static_cast<uint32_t>(last_active + 1);
    for (int b = 0; b < L::kNumBars; ++b) {
      const bool p_bar = (b == BAR_P_FULL || b == BAR_P_FULL + 1);
      const bool kv_bar = b == BAR_K_EMPTY || b == BAR_K_EMPTY + 1 || b == BAR_V_EMPTY || b == BAR_V_EMPTY + 1;
      mbar_init(bar(b), p_bar ? 128u : ((b == BAR_DRAIN || (SHARED && kv_bar)) ? n_issuers : 1u));
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (PAIR && (warp == 10 || warp == 11)) {
    // warp 10 builds slot 0's union list, warp 11 slot 1's
    const int h = warp - 10;
    const Slot& sl = h ? slot[1] : slot[0];
    int len = 0;
    if (sl.active) {
      const int32_t* row_a = a.idx + (static_cast<size_t>(sl.bh) * g.nT + sl.tile) * a.topk;
      const int nw = L::bitmap_words(gk.nT);
      len = build_union<SAME>(a, row_a, sl.has_b, bitmaps + 2 * h * nw, bitmaps + (2 * h + 1) * nw,
                        unions + h * 2 * a.topk);
    }
    if (lane == 0) union_len[h] = len;
  }
  if (PAIR) {
    // a slot without tile B (odd tile count) computes rows 64-127 from zeros
    for (int h = 0; h < 2; ++h) {
      if (!slot[h].active || slot[h].has_b) continue;
      for (int sl = 0; sl < L::kSlabs; ++sl) {
        uint4* q4 = reinterpret_cast<uint4*>(sp + L::kQ + h * L::kBufBytes + sl * L::kSlabBytes + 64 * 128);
        for (int e = threadIdx.x; e < 64 * 128 / 16; e += kAttnThreads) q4[e] = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    setmaxnreg_dec<RegSplit<MODE>::kProducer>();
  }
  if (warp == 8 || (!SHARED && warp == 11)) {
    // ====================================================== TMA producer(s)
    // MODE_SHARED streams one K/V sequence for both slots (warp 8).  In
    // MODE_TILE and MODE_PAIR each slot owns one K and one V stage and warp 8
    // serves slot 0, warp 11 slot 1: with one producer for both, a slot's next
    // K waited behind the other slot's V release (LongCat-like: the MMA issuer
    // waited ~1300 clk for K after P was ready).
    const int h_only = SHARED ? -1 : (warp == 8 ? 0 : 1);
    if (lane == 0) {
      bool ok = true;
      for (int h = 0; h < 2; ++h) {
        if (!slot[h].active || (h_only >= 0 && h != h_only)) continue;
        const int nbox = (PAIR && slot[h].has_b) ? 2 : 1;
        mbar_arrive_expect_tx(bar(BAR_Q_FULL + h), static_cast<uint32_t>(nbox * L::kSlabs) * box_bytes);
        const BoxCoord ca = box_coord_l<BNHD>(g, slot[h].bh, slot[h].t0, slot[h].y0, slot[h].x0);
        const BoxCoord cb = box_coord_l<BNHD>(g, slot[h].bh, slot[h].tb0, slot[h].yb0, slot[h].xb0);
        for (int sl = 0; sl < L::kSlabs; ++sl) {
          tma_load_5d(sQ + h * L::kBufBytes + sl * L::kSlabBytes, &tmQ, bar(BAR_Q_FULL + h), sl * 64, ca.c1,
                      ca.c2, ca.c3, ca.c4);
          if (nbox == 2)
            tma_load_5d(sQ + h * L::kBufBytes + sl * L::kSlabBytes + box_bytes, &tmQ, bar(BAR_Q_FULL + h),
                        sl * 64, cb.c1, cb.c2, cb.c3, cb.c4);
        }
      }
      KvSeq<MODE, SAME> sq[2];
      int n[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        sq[h].init(a, tile_tab, slot[h].bh, slot[h].tile, unions + h * 2 * a.topk, union_len[h]);
        n[h] = slot[h].active ? sq[h].count(a) : 0;
      }
      const int n_max = SHARED ? n[0] : max(n[0], n[1]);
      int last_use[2][2] = {{-1, -1}, {-1, -1}};   // [K/V][stage]: last phase issued
      for (int it = 0; it < n_max && ok; ++it) {
        for (int kv = 0; kv < 2 && ok; ++kv) {         // K first, then V
          const CUtensorMap* tm = kv == 0 ? &tmK : &tmV;
          const uint32_t buf0 = kv == 0 ? sK : sV;
          const int full = kv == 0 ? BAR_K_FULL : BAR_V_FULL;
          const int empty = kv == 0 ? BAR_K_EMPTY : BAR_V_EMPTY;
#pragma unroll
          for (int h = 0; h < (SHARED ? 1 : 2); ++h) {
            if (!ok || it >= n[h] || (h_only >= 0 && h != h_only)) continue;
            const int st = SHARED ? (it & 1) : h;
            const int use = SHARED ? (it >> 1) : it;
            if (use > 0 && !mbar_wait(bar(empty + st), (use - 1) & 1, abort_flag, a.err)) {
              ok = false;
              continue;
            }
            mbar_arrive_expect_tx(bar(full + st), static_cast<uint32_t>(P * L::kSlabs) * box_bytes);
            last_use[kv][st] = use;
#pragma unroll
            for (int p = 0; p < P; ++p) {
              const Piece pc = sq[h].piece(a, p, kv == 0);
              const TileCoord c = table_coord(tile_tab, pc.j);
              const BoxCoord bc =
                  box_coord_l<BNHD>(gk, slot[h].bh, c.bt * gk.tt + pc.toff, c.by * gk.th, c.bx * gk.tw);
              for (int sl = 0; sl < L::kSlabs; ++sl)
                tma_load_5d(buf0 + st * L::kBufBytes + sl * L::kSlabBytes + p * box_bytes, tm,
                            bar(full + st), sl * 64, bc.c1, bc.c2, bc.c3, bc.c4);
            }
          }
        }
        sq[0].advance(a);
        sq[1].advance(a);
      }
      // Let every issued copy land before the CTA can exit (returns at once
      // when the consumers already saw these phases complete).
      for (int kv = 0; kv < 2; ++kv)
        for (int st = 0; st < 2; ++st)
          if (last_use[kv][st] >= 0)
            mbar_wait(bar((kv == 0 ? BAR_K_FULL : BAR_V_FULL) + st), last_use[kv][st] & 1, nullptr, a.err);
    }
    __syncwarp();
  } else if (warp == 9 || warp == 10) {
    // ====================================================== MMA issuer(s)
    constexpr uint32_t idS = idesc_f16kind_f32(kSlotRows, kSubRows, false, F16);
    constexpr uint32_t idPV = idesc_f16kind_f32(kSlotRows, D, true, F16);
    // Operand descriptors.  MODE_SHARED holds three and adds (byte offset >>
    // 4): the address field keeps shared-memory addresses >> 4 in 14 bits,
    // and every address here is 16-byte aligned and below 256 KB, so the sum
    // never carries out of it (2 % faster there; the other modes have no
    // registers to spare and build each descriptor in place).
    const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
    const uint64_t dK = smem_desc_sw128(sK, 16, 1024);
    const uint64_t dV = smem_desc_sw128(sV, L::kSlabBytes, 1024);
    auto desc_qk = [&](uint64_t d0, uint32_t s0, int buf, int kk) -> uint64_t {
      const int sl = kk / 4, koff = (kk % 4) * 32;        // 16 channels = 32 B within a 64-channel slab
      const uint32_t off = static_cast<uint32_t>(buf * L::kBufBytes + sl * L::kSlabBytes + koff);
      return SHARED ? d0 + (off >> 4) : smem_desc_sw128(s0 + off, 16, 1024);
    };
    auto issue_pv = [&](int h, int vst, bool acc) {
      const uint32_t tS = tmem + 128u * h, tO = tmem + 256u + 128u * h;
#pragma unroll
      for (int kk = 0; kk < kSubRows / 16; ++kk) {        // 16 keys = 16 rows of 128 B
        const uint32_t off = static_cast<uint32_t>(vst * L::kBufBytes + kk * 2048);
        const uint64_t bd = SHARED ? dV + (off >> 4) : smem_desc_sw128(sV + off, L::kSlabBytes, 1024);
        mma_ts(tO, tS + 8u * kk, bd, idPV, (acc || kk > 0) ? 1u : 0u);
      }
    };
    auto issue_s = [&](int h, int kst) {
      const uint32_t tS = tmem + 128u * h;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tS, desc_qk(dQ, sQ, h, kk), desc_qk(dK, sK, kst, kk), idS, kk > 0 ? 1u : 0u);
    };

    // One issuer warp per slot (warp 9 + h), whole warp in the loop (waits,
    // counters and descriptors are warp-uniform), one elected lane issuing
    // each group and its commits (a commit tracks the MMAs of the thread that
    // issued them; the warp is converged at every election, so it is always
    // the same lane).  After a thread queues MMAs, its own next shared-memory
    // access -- a barrier test included -- waits until that queue has nearly
    // drained, so a single issuer for both slots would see slot 1's P only
    // when slot 0's S is almost done and leave the tensor pipe idle while it
    // catches up.  Here each warp tests its own slot's barriers with an empty
    // queue.  The two warps pass a token through named barriers 1 and 2 (which
    // do not wait for the MMA queue), so the groups still enter the pipe in
    // the order PV_0, S_0, PV_1, S_1: groups of two issuers left free to
    // interleave finish later for both slots.  Both warps take the same
    // n_max + 1 token steps whatever happens (a failed wait, or a slot with
    // fewer sub-blocks, only skips the MMAs), so neither can be left waiting
    // at a named barrier.  In MODE_SHARED both issuers release each K/V stage
    // (barrier count = active slots); otherwise a stage belongs to one slot.
    {
      const int h = warp - 9;
      int nn[2];
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        KvSeq<MODE, SAME> sq2;
        sq2.init(a, tile_tab, slot[s2].bh, slot[s2].tile, unions + s2 * 2 * a.topk, union_len[s2]);
        nn[s2] = slot[s2].active ? sq2.count(a) : 0;
      }
      const int n = h ? nn[1] : nn[0];
      const int n_max = max(nn[0], nn[1]);
      if (slot[h].active) {
        const bool token = last_active == 1;           // two issuers
        bool ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_Q_FULL + h), 0, abort_flag, a.err));
        for (int it = 0; it <= n_max; ++it) {
          if (token) {
            if (h == 1) named_bar_sync(1, 64);
            else if (it > 0) named_bar_sync(2, 64);
          }
          const int kst = SHARED ? (it & 1) : h, kpar = SHARED ? ((it >> 1) & 1) : (it & 1);
          const int vst = SHARED ? ((it - 1) & 1) : h, vpar = SHARED ? (((it - 1) >> 1) & 1) : ((it - 1) & 1);
          if (it > n) { if (token) named_bar_arrive(h == 0 ? 1 : 2, 64); continue; }
          if (ok && it < n) ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_K_FULL + kst), kpar, abort_flag, a.err));
          if (ok && it > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_P_FULL + h), (it - 1) & 1, abort_flag, a.err) &&
                                             mbar_wait(bar(BAR_V_FULL + vst), vpar, abort_flag, a.err));
          if (ok) {
            tc_fence_after();
            if (elect_one_sync()) {
              if (it > 0) {
                issue_pv(h, vst, it - 1 > 0);
                mma_commit(bar(it == n ? BAR_O_FULL + h : BAR_V_EMPTY + vst));
              }
              if (it < n) {
                issue_s(h, kst);
                mma_commit(bar(BAR_S_FULL + h));
                mma_commit(bar(BAR_K_EMPTY + kst));
              }
            }
            __syncwarp();
          }
          if (token) named_bar_arrive(h == 0 ? 1 : 2, 64);
        }
        if (token && h == 0) named_bar_sync(2, 64);    // warp 10's last arrival
        // Drain: every MMA of both issuers has finished before TMEM is freed.
        if (elect_one_sync()) mma_commit(bar(BAR_DRAIN));
        __syncwarp();
        mbar_wait(bar(BAR_DRAIN), 0, nullptr, a.err);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ====================================================== softmax slot h
    setmaxnreg_inc<RegSplit<MODE>::kSoftmax>();
    const int h = warp / 4;
    const int q = warp % 4;
    const int r = threadIdx.x % 128;                  // query row of the slot = TMEM lane
    Slot me;                                          // slot[h] without run-time indexing
    me.active = h ? slot[1].active : slot[0].active;
    me.bh = h ? slot[1].bh : slot[0].bh;
    me.tile = h ? slot[1].tile : slot[0].tile;
    me.has_b = h ? slot[1].has_b : slot[0].has_b;
    // MODE_PAIR: rows 64-127 (warps 2-3 of the warpgroup) belong to tile B
    const bool in_b = PAIR && r >= 64;
    me.t0 = in_b ? (h ? slot[1].tb0 : slot[0].tb0) : (h ? slot[1].t0 : slot[0].t0);
    me.y0 = in_b ? (h ? slot[1].yb0 : slot[0].yb0) : (h ? slot[1].y0 : slot[0].y0);
    me.x0 = in_b ? (h ? slot[1].xb0 : slot[0].xb0) : (h ? slot[1].x0 : slot[0].x0);
    if (me.active) {
      const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
      const uint32_t tS = tmem + lane_base + 128u * h;
      const uint32_t tO = tmem + lane_base + 256u + 128u * h;
      const int lg_yx = g.lg_th + g.lg_tw;
      const int lg_yx_k = gk.lg_th + gk.lg_tw;

      // which token this row is (if any)
      bool row_valid;
      int tok_t, tok_y, tok_x;
      {
        const int rr = PAIR ? (r & 63) : r;
        const int lt = rr >> lg_yx, ly = (rr >> g.lg_tw) & (g.th - 1), lx = rr & (g.tw - 1);
        tok_t = me.t0 + lt;
        tok_y = me.y0 + ly;
        tok_x = me.x0 + lx;
        row_valid = rr < box_rows && tok_t < g.T && tok_y < g.Hh && tok_x < g.W &&
                    lt < (SHARED ? a.box_tq : g.tt) && (!in_b || me.has_b);
      }

      KvSeq<MODE, SAME> sq;
      sq.init(a, tile_tab, me.bh, me.tile, unions + h * 2 * a.topk, union_len[h]);
      const int n = sq.count(a);
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int it = 0; it < n; ++it) {
        // Which key columns count for this warp's rows: columns [0, 64) are
        // piece 0 and [64, 128) piece 1 (one 128-column piece outside
        // MODE_PAIR).  use0/use1: the piece was kept by this row's query tile
        // (warp-uniform); a piece that is not used contributes P = 0 without
        // any exponential.  Partial tiles at the grid edge need a column mask.
        uint32_t mw[4] = {~0u, ~0u, ~0u, ~0u};
        bool use0 = true, use1 = true, geo_full = true;
        {
          int vt0 = 0, vy0 = 0, vx0 = 0, vt1 = 0, vy1 = 0, vx1 = 0;
#pragma unroll
          for (int p = 0; p < P; ++p) {
            const Piece pc = sq.piece(a, p, false);
            const TileCoord c = table_coord(tile_tab, pc.j);
            int et, ey, ex;
            tile_extent(gk, c, et, ey, ex);
            const int vt = SHARED ? min(kv_box_t<SAME>(a), et - pc.toff) : et;
            const bool use = pc.real && (in_b ? pc.in_b : pc.in_a);
            const bool gfull = vt == (SHARED ? kv_box_t<SAME>(a) : gk.tt) && ey == gk.th && ex == gk.tw;
            geo_full = geo_full && (!use || gfull);
            if (p == 0) { vt0 = vt; vy0 = ey; vx0 = ex; use0 = use; }
            else        { vt1 = vt; vy1 = ey; vx1 = ex; use1 = use; }
          }
          if (!PAIR) use1 = use0;
          if (!geo_full) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int col = 32 * w + lane;
              const bool second = PAIR && col >= gk.vol;
              const int rr = second ? col - gk.vol : col;
              const int lt = rr >> lg_yx_k, ly = (rr >> gk.lg_tw) & (gk.th - 1), lx = rr & (gk.tw - 1);
              const bool v = second ? (use1 && lt < vt1 && ly < vy1 && lx < vx1)
                                    : (use0 && lt < vt0 && ly < vy0 && lx < vx0);
              mw[w] = __ballot_sync(0xffffffffu, v);
            }
          }
        }
        sq.advance(a);

        if (!__all_sync(0xffffffffu, mbar_wait(bar(BAR_S_FULL + h), it & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[128];
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
        tmem_wait_ld();

        if (!geo_full) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = __float_as_uint(-INFINITY);
        }
        // row max over the used halves, each a tree of 4 chains of 3-input max
        float mxh[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!(hf ? use1 : use0)) continue;
          float mx4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) mx4[e] = __uint_as_float(s[64 * hf + e]);
#pragma unroll
          for (int c = 64 * hf + 4; c < 64 * hf + 64; c += 2)
            mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          mxh[hf] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        }
        const float mx_s = fmaxf(mxh[0], mxh[1]) * a.scale_log2;

        // lazy rescale: move the reference max only when it grew by > 2^8.  A
        // row may see no valid key in a sub-block (mx = -inf, MODE_PAIR); its
        // reference stays -inf until one arrives, with 0 used in the exponent.
        float alpha = 1.f;
        if (mx_s > m + kRescaleLog2) {
          alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - mx_s);
          m = mx_s;
          l *= alpha;
        }
        const bool rescale = __any_sync(0xffffffffu, alpha != 1.f) && it > 0;
        const float m_use = (m == -INFINITY) ? 0.f : m;
        // P = 2^(scale*log2(e)*S - m) on pairs of columns; row sum in 4 packed chains
        const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
        const uint64_t nm2 = f2_pack(-m_use, -m_use);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!(hf ? use1 : use0)) {
#pragma unroll
            for (int c = 32 * hf; c < 32 * hf + 32; ++c) s[c] = 0u;     // P = 0
            tmem_st32(tS + 32u * hf, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * hf]));
            continue;
          }
#pragma unroll
          for (int c = 32 * hf; c < 32 * hf + 32; ++c) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), sc2, nm2);
            float p0, p1;
            if ((c & 7) < kExpPolyPer8) {
              exp2_poly_pair(x2, p0, p1);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            ls2[c & 3] = f2_add(ls2[c & 3], f2_pack(p0, p1));
            s[c] = (kPackAlu && !F16) ? pack_bf16x2_alu(p0, p1) : pack_elem2<F16>(p0, p1);
          }
          // store each half of P as soon as it is packed: the first store
          // overlaps the second half's exponentials
          tmem_st32(tS + 32u * hf, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * hf]));
        }
        {
          float a0, a1;
          f2_unpack(f2_add(f2_add(ls2[0], ls2[1]), f2_add(ls2[2], ls2[3])), a0, a1);
          l += a0 + a1;
        }
        if (rescale) {
          // O_h is idle here: PV_h(it-1) completed before S_h(it) did, and
          // PV_h(it) waits for this slot's P_FULL arrival below.
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t ov[32];
            tmem_ld32(tO + 32u * c4, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tO + 32u * c4, ov);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(BAR_P_FULL + h));
      }

      // ---- epilogue: O / l -> the input type, LSE
      if (ok && __all_sync(0xffffffffu, mbar_wait(bar(BAR_O_FULL + h), 0, abort_flag, a.err))) {
        tc_fence_after();
        const float inv_l = 1.f / l;
        const size_t N = static_cast<size_t>(g.T) * g.Hh * g.W;
        const size_t n_tok = (static_cast<size_t>(tok_t) * g.Hh + tok_y) * g.W + tok_x;
        uint16_t* orow = a.o + token_offset(g, me.bh, n_tok);
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t ov[32];
          tmem_ld32(tO + 32u * c4, ov);
          tmem_wait_ld();
          if (row_valid) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_elem2<F16>(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
            // streaming stores: O is not read again by this kernel, so it
            // should not sit dirty in L2 for whatever kernel runs next
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c4);
#pragma unroll
            for (int e = 0; e < 4; ++e) __stcs(dst + e, make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]));
          }
        }
        if (row_valid)
          __stcs(a.lse + static_cast<size_t>(me.bh) * N + n_tok, (m + log2f(l)) * 0.69314718055994530942f);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace vsa
