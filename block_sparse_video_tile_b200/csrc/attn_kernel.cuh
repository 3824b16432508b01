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
// One CTA = one "slot" of 128 query rows (MMA M = 128):
//   MODE_SHARED (tiles of 256 tokens, tt >= 2): one t-half of a query tile;
//     a K/V sub-block is a t-half of a kept tile (the two t-halves of a query
//     tile are neighbouring CTAs, so they share their K/V reads in L2).
//   MODE_TILE (tiles of 128 tokens): one query tile; a K/V sub-block is one
//     of its kept tiles.
//   MODE_PAIR (tiles of 64 tokens): two neighbouring query tiles A (rows
//     0-63) and B (rows 64-127).  The slot walks the union of their kept
//     lists, two 64-token tiles per K/V sub-block, and every row masks the
//     tiles only the other query tile kept.  Neighbouring tiles of a video
//     keep mostly the same tiles, so most of each 128-row MMA is useful work;
//     at worst (disjoint lists) it is half, as with one padded tile.
// Warp roles (384 threads): two softmax warpgroups, warps 0-3 and 4-7, both
// on the slot's 128 rows (thread = query row = TMEM lane), warpgroup w taking
// the sub-blocks it with it % 2 == w, so two warps per SM sub-partition hide
// each other's latencies and each has two sub-block periods for its work;
// thread 0 issues Q's TMA load as soon as the barriers exist (it overlaps the
// rest of the set-up), warp 8 loads the K stream by TMA, warp 9 the V stream
// (and in MODE_PAIR first builds the union list), warp 10 issues the PV MMAs
// and warp 11 the score MMAs (tcgen05.mma kind::f16, float32 accumulation);
// the third warpgroup gives registers to the softmax (setmaxnreg).
// TMEM (512 columns): three score buffers of 128 columns and O at 384.  The
// scores of sub-block it go to buffer it % 3 and the softmax writes P (16-bit
// pairs, 64 columns) over them; PV(it) reads P from there, and S(it+3) goes
// into the same buffer once PV(it) has completed (S_FREE).  So the scores of
// the next two sub-blocks are computed while the softmax works on this one:
// the softmax never waits for its own MMAs, and the tensor pipe waits only
// for P.  The PV and score MMAs have an issuing warp each: a thread that has
// queued MMAs sees its next shared-memory access (a barrier test included)
// wait until that queue has nearly drained, so one issuer for both would
// notice a stored P only after the scores queued ahead of it (measured
// ~750 clk late).  Every MMA is a full 128 x 128 x 16 step (narrower N costs about as
// much per instruction: 57 clk at N = 64 against 64 at N = 128, measured).
// Online softmax in float32 with lazy rescaling (O and l are rescaled only
// when the running max grows by more than 2^8).  The two warpgroups share the
// row's reference max in order: each computes its sub-block's exponentials
// against the reference it last knew, then takes the settled value of the
// sub-block before from shared memory (M_READY), settles its own and passes
// it on; when the other warpgroup moved the reference meanwhile (rare), it
// rescales the P it already stored.
// Epilogue: O / l (plus the gated coarse term) in the input type is staged in
// the Q buffer, swizzled as the Q boxes arrived, and written by one TMA store
// per box and slab; the output map keeps every box inside its batch, so the
// stores drop the rows past the grid edge.  LSE goes out by plain stores.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "vsa_geometry.cuh"
#include "vsa_ptx.cuh"

namespace vsa {

constexpr int kAttnThreads = 384;       // 3 warpgroups
constexpr int kWarpK = 8, kWarpV = 9, kWarpPV = 10, kWarpS = 11;
// Registers per thread after setmaxnreg: softmax warpgroups and the third
// (TMA and MMA warps).  2*128*S + 128*P must stay within the launch's 384*168.
template <int MODE>
struct RegSplit {
  static constexpr int kSoftmax = MODE == 2 ? 200 : 208;
  static constexpr int kProducer = MODE == 2 ? 96 : 88;
  static_assert(2 * 128 * kSoftmax + 128 * kProducer <= 384 * 168, "register split over the launch budget");
};
constexpr int kSlotRows = 128;          // MMA M
constexpr int kSubRows = 128;           // K/V rows per sub-block (S: N, PV: K)
constexpr int kSBufs = 3;               // score buffers in TMEM
constexpr uint32_t kTmemO = 384;        // TMEM column of O
constexpr float kRescaleLog2 = 8.0f;
#ifndef VSA_EXP_POLY_PER8
#define VSA_EXP_POLY_PER8 0
#endif
// Of every 8 column pairs of a score row, this many take 2^x on the FMA pipe
// (exp2_poly_pair) and the rest on the multi-function unit (ex2.approx): the
// two units then share the softmax's exponentials.
constexpr int kExpPolyPer8 = VSA_EXP_POLY_PER8;
constexpr uint32_t kErrBadIndex = 2u;
constexpr uint32_t kErrBadOrder = 3u;

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
  // pooled coarse branch (both or neither): O += gate * coarse[query tile]
  const uint16_t* gate;      // Q's layout and type, or nullptr
  const float* coarse;       // [B*H, nTq, d] float32
};

template <int D>
struct AttnSmem {
  static constexpr int kSlabBytes = 128 * 128;       // 128 rows x 64 bf16 (one 128B-swizzle slab)
  static constexpr int kSlabs = D / 64;
  static constexpr int kBufBytes = kSlabs * kSlabBytes;
  static constexpr int kQ = 0;                        // 1 buffer
  static constexpr int kK = kBufBytes;                // 2 stages
  static constexpr int kV = 3 * kBufBytes;            // 2 stages
  static constexpr int kBar = 5 * kBufBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kMisc = kBar + kNumBars * 8;   // TMEM address, abort flag, union length
  static constexpr int kRows = kMisc + 16;            // float [3][2][128]: settled max per sub-block parity,
                                                      // and each warpgroup's final (l, m) for the epilogue
  static constexpr int kTiles = kRows + 3 * 2 * 128 * 4;   // uint2 per tile: (bt, by | bx << 16)
  // then the slot's list: MODE_PAIR: membership bitmaps (2 x ceil(nT/32)
  // words) and the union list (up to 2*topk entries of j | in_a << 16 |
  // in_b << 17); otherwise the kept tiles (topk entries)
  __host__ __device__ static int bitmap_off(int nT) { return kTiles + ((8 * nT + 15) & ~15); }
  __host__ __device__ static int bitmap_words(int nT) { return (nT + 31) / 32; }
  __host__ __device__ static int union_off(int nT) { return bitmap_off(nT) + ((8 * bitmap_words(nT) + 15) & ~15); }
  // then one uint2 per K/V sub-block (at most 2*topk): what the softmax
  // needs of it (see sub_desc)
  __host__ __device__ static int desc_off(int nT, int topk) { return union_off(nT) + ((2 * topk * 4 + 15) & ~15); }
  __host__ __device__ static int total(int nT, int topk, bool pair) { return desc_off(nT, topk) + 2 * topk * 8; }
  __host__ __device__ static int alloc(int nT, int topk, bool pair) { return total(nT, topk, pair) + 1024; }
};

// mbarriers.  S_FULL[b]: scores in buffer b; P_FULL[b]: P stored over them
// (and O rescaled if it had to be); S_FREE[b]: the PV that read buffer b has
// completed; PV_DONE[x]: PV of the sub-blocks of parity x, one phase each, in
// order; M_READY[x]: the settled reference max of a sub-block of parity x is
// in shared memory; O_FULL: the last PV; DRAIN: both issuers' MMAs are done.
enum : int {
  BAR_Q_FULL = 0, BAR_K_FULL = 1, BAR_K_EMPTY = 3, BAR_V_FULL = 5, BAR_V_EMPTY = 7,
  BAR_S_FULL = 9, BAR_P_FULL = 12, BAR_PV_DONE = 15, BAR_M_READY = 17, BAR_O_FULL = 19, BAR_DRAIN = 20,
  BAR_S_FREE = 21
};

// The CTA's query rows: head, query tile (tile A in MODE_PAIR) and the origin
// of its box (and of tile B's).
struct Slot {
  bool active;
  int bh, tile;
  int t0, y0, x0;
  bool has_b;            // MODE_PAIR: tile B = tile + 1 exists
  int tb0, yb0, xb0;
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

// K/V sub-block sequence of the slot, read from its list in shared memory
// (copied from idx and checked at kernel start, so the loop never waits on
// global memory for it).
//   MODE_SHARED: for each kept tile (ascending), its t-halves that hold a token.
//   MODE_TILE:   each kept tile.
//   MODE_PAIR:   the ascending union of tile A's and tile B's kept lists
//                (entries j | in_a << 16 | in_b << 17), two tiles per
//                sub-block (a short last sub-block is padded).
template <int MODE, bool SAME>
struct KvSeq {
  const uint32_t* list;   // kept tiles (MODE_PAIR: the union list), shared memory
  int len;                // entries in list
  const uint2* tab;
  int pos, half;

  __device__ void init(const uint2* table, const uint32_t* l, int n) {
    list = l;
    len = n;
    tab = table;
    pos = 0;
    half = 0;
  }
  __device__ bool second_half(const AttnArgs& a, int j) const {
    return static_cast<int>(tab[j].x) * kv_geom<SAME>(a).tt + kv_box_t<SAME>(a) < kv_geom<SAME>(a).T;
  }
  __device__ int count(const AttnArgs& a) const {
    if (MODE == MODE_TILE) return len;
    if (MODE == MODE_PAIR) return (len + 1) / 2;
    int n = 0;
    for (int e = 0; e < len; ++e) n += 1 + (second_half(a, static_cast<int>(list[e])) ? 1 : 0);
    return n;
  }
  // Piece p (0 or 1) of the current sub-block.
  __device__ Piece piece(const AttnArgs& a, int p) const {
    Piece pc;
    if (MODE == MODE_SHARED) {
      pc.j = static_cast<int>(list[pos]);
      pc.toff = half * kv_box_t<SAME>(a);
      pc.real = pc.in_a = pc.in_b = true;
    } else if (MODE == MODE_TILE) {
      pc.j = static_cast<int>(list[pos]);
      pc.toff = 0;
      pc.real = pc.in_a = pc.in_b = true;
    } else {
      const int e = 2 * pos + p;
      const bool real = e < len;
      const uint32_t u = list[real ? e : 2 * pos];   // padding repeats a real piece, all masked
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
      if (half == 0 && pos < len && second_half(a, static_cast<int>(list[pos]))) {
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

// Per K/V sub-block, what the softmax needs: x = vt0 | vy0 << 8 | vx0 << 16
// | flags << 24, y = vt1 | vy1 << 8 | vx1 << 16, with (vt, vy, vx) the valid
// extents of piece 0 / 1 and flags: 1, 2 = piece 0 kept by query tile A, B;
// 4, 8 = piece 1 kept by A, B; 16, 32 = piece 0, 1 is a full box (no mask).
// Written once per CTA by one warp, so the softmax loop reads one shared
// memory word pair per sub-block instead of walking the kept list.
template <int MODE, bool SAME>
__device__ __forceinline__ uint32_t piece_word(const AttnArgs& a, const uint2* tab, const Piece& pc, bool& full) {
  const TileCoord c = table_coord(tab, pc.j);
  int et, ey, ex;
  tile_extent(kv_geom<SAME>(a), c, et, ey, ex);
  const int vt = MODE == MODE_SHARED ? min(kv_box_t<SAME>(a), et - pc.toff) : et;
  full = vt == (MODE == MODE_SHARED ? kv_box_t<SAME>(a) : kv_geom<SAME>(a).tt) && ey == kv_geom<SAME>(a).th &&
         ex == kv_geom<SAME>(a).tw;
  return static_cast<uint32_t>(vt) | (static_cast<uint32_t>(ey) << 8) | (static_cast<uint32_t>(ex) << 16);
}

template <int MODE, bool SAME>
__device__ __forceinline__ void build_sub_desc(const AttnArgs& a, const uint2* tab, const uint32_t* list, int len,
                                               uint2* desc) {
  const int lane = threadIdx.x % 32;
  auto write = [&](int sidx, const Piece& p0, const Piece& p1) {
    bool f0, f1;
    const uint32_t w0 = piece_word<MODE, SAME>(a, tab, p0, f0);
    const uint32_t w1 = piece_word<MODE, SAME>(a, tab, p1, f1);
    const uint32_t fl = (p0.real && p0.in_a ? 1u : 0u) | (p0.real && p0.in_b ? 2u : 0u) |
                        (p1.real && p1.in_a ? 4u : 0u) | (p1.real && p1.in_b ? 8u : 0u) | (f0 ? 16u : 0u) |
                        (f1 ? 32u : 0u);
    desc[sidx] = make_uint2(w0 | (fl << 24), w1);
  };
  if (MODE == MODE_SHARED) {
    // kept tile e gives one or two sub-blocks (its t-halves that hold a
    // token): positions by a prefix count across the warp
    int base = 0;
    for (int e0 = 0; e0 < len; e0 += 32) {
      const int e = e0 + lane;
      const int j = e < len ? static_cast<int>(list[e]) : 0;
      const bool two = e < len &&
                       static_cast<int>(tab[j].x) * kv_geom<SAME>(a).tt + kv_box_t<SAME>(a) < kv_geom<SAME>(a).T;
      const int cnt = e < len ? (two ? 2 : 1) : 0;
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      for (int hh = 0; hh < cnt; ++hh) {
        Piece pc;
        pc.j = j;
        pc.toff = hh * kv_box_t<SAME>(a);
        pc.real = pc.in_a = pc.in_b = true;
        write(base + incl - cnt + hh, pc, pc);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
  } else if (MODE == MODE_TILE) {
    for (int e = lane; e < len; e += 32) {
      Piece pc;
      pc.j = static_cast<int>(list[e]);
      pc.toff = 0;
      pc.real = pc.in_a = pc.in_b = true;
      write(e, pc, pc);
    }
  } else {
    for (int sb = lane; 2 * sb < len; sb += 32) {
      Piece pc[2];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int e = 2 * sb + p;
        const bool real = e < len;
        const uint32_t u = list[real ? e : 2 * sb];   // padding repeats a real piece, all masked
        pc[p].j = static_cast<int>(u & 0xffffu);
        pc[p].toff = 0;
        pc[p].real = real;
        pc[p].in_a = real && ((u >> 16) & 1u);
        pc[p].in_b = real && ((u >> 17) & 1u);
      }
      write(sb, pc[0], pc[1]);
    }
  }
}

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
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const AttnArgs a) {
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
  int* union_len = reinterpret_cast<int*>(sp + L::kMisc + 8);
  uint2* tile_tab = reinterpret_cast<uint2*>(sp + L::kTiles);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(sp + L::bitmap_off(kv_geom<SAME>(a).nT));
  uint32_t* unions = reinterpret_cast<uint32_t*>(sp + L::union_off(kv_geom<SAME>(a).nT));
  uint2* sub_desc = reinterpret_cast<uint2*>(sp + L::desc_off(kv_geom<SAME>(a).nT, a.topk));
  auto bar = [&](int id) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(id); };

  const Geom& g = a.gq;                                     // query side
  const Geom& gk = kv_geom<SAME>(a);                        // key/value side
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int box_rows = SHARED ? kSubRows : g.vol;          // rows per TMA box (equal volumes)
  const uint32_t box_bytes = static_cast<uint32_t>(box_rows) * 128u;

  // ---- work unit -> the CTA's query rows
  Slot slot;
  {
    int bh, tile, toff = 0;
    bool has_b = false;
    if (SHARED) {                                            // (head, tile, t-half)
      const int u = static_cast<int>(blockIdx.x);
      bh = u / (2 * g.nT);
      tile = (u / 2) % g.nT;
      toff = (u & 1) * a.box_tq;
    } else if (MODE == MODE_TILE) {
      bh = static_cast<int>(blockIdx.x) / g.nT;
      tile = static_cast<int>(blockIdx.x) % g.nT;
    } else {
      const int npair = (g.nT + 1) / 2;
      bh = static_cast<int>(blockIdx.x) / npair;
      tile = 2 * (static_cast<int>(blockIdx.x) % npair);
      has_b = tile + 1 < g.nT;
    }
    const TileCoord c = tile_coord(g, tile);
    slot.bh = bh;
    slot.tile = tile;
    slot.t0 = c.bt * g.tt + toff;
    slot.y0 = c.by * g.th;
    slot.x0 = c.bx * g.tw;
    slot.active = slot.t0 < g.T;
    slot.has_b = has_b;
    const TileCoord cb = tile_coord(g, has_b ? tile + 1 : tile);
    slot.tb0 = cb.bt * g.tt;
    slot.yb0 = cb.by * g.th;
    slot.xb0 = cb.bx * g.tw;
  }
  if (!slot.active) return;                                  // (a t-half past the last frame)

  // ---- setup: tile table, kept-list check, barriers, union list, TMEM
  for (int j = threadIdx.x; j < gk.nT; j += kAttnThreads) {
    const TileCoord c = tile_coord(gk, j);
    tile_tab[j] = make_uint2(static_cast<uint32_t>(c.bt),
                             static_cast<uint32_t>(c.by) | (static_cast<uint32_t>(c.bx) << 16));
  }
  // The slot's kept lists must be strictly ascending (as tile selection writes
  // them): a row that is not is reported in the error word (the CTA still
  // runs with every load in bounds; that row's result is unspecified).
  {
    const int rows = (PAIR && slot.has_b) ? 2 : 1;
    const int32_t* r0 = a.idx + (static_cast<size_t>(slot.bh) * g.nT + slot.tile) * a.topk;
    for (int e = threadIdx.x; e < rows * a.topk; e += kAttnThreads)
      if (e % a.topk != 0 && __ldg(r0 + e) <= __ldg(r0 + e - 1)) atomicCAS(a.err, 0u, kErrBadOrder);
  }
  if (threadIdx.x == 0) {
    for (int b = 0; b < L::kNumBars; ++b) {
      // one arrival per thread of the softmax warpgroup taking the sub-block
      const bool p_bar = (b >= BAR_P_FULL && b < BAR_P_FULL + kSBufs) || b == BAR_M_READY || b == BAR_M_READY + 1;
      mbar_init(bar(b), p_bar ? 128u : (b == BAR_DRAIN ? 2u : 1u));
    }
    *abort_flag = 0;
    fence_mbar_init();
    // Q needs nothing of the set-up below: its load overlaps it
    const int nbox = (PAIR && slot.has_b) ? 2 : 1;
    mbar_arrive_expect_tx(bar(BAR_Q_FULL), static_cast<uint32_t>(nbox * L::kSlabs) * box_bytes);
    const BoxCoord ca = box_coord_l<BNHD>(g, slot.bh, slot.t0, slot.y0, slot.x0);
    const BoxCoord cb = box_coord_l<BNHD>(g, slot.bh, slot.tb0, slot.yb0, slot.xb0);
    for (int sl = 0; sl < L::kSlabs; ++sl) {
      tma_load_5d(sQ + sl * L::kSlabBytes, &tmQ, bar(BAR_Q_FULL), sl * 64, ca.c1, ca.c2, ca.c3, ca.c4);
      if (nbox == 2)
        tma_load_5d(sQ + sl * L::kSlabBytes + box_bytes, &tmQ, bar(BAR_Q_FULL), sl * 64, cb.c1, cb.c2, cb.c3, cb.c4);
    }
  }
  if (!PAIR) {
    const int32_t* r0 = a.idx + (static_cast<size_t>(slot.bh) * g.nT + slot.tile) * a.topk;
    for (int e = threadIdx.x; e < a.topk; e += kAttnThreads)
      unions[e] = static_cast<uint32_t>(load_tile_index<SAME>(a, r0, e, true));
  }
  if (PAIR && warp == kWarpV) {
    int len = 0;
    const int32_t* row_a = a.idx + (static_cast<size_t>(slot.bh) * g.nT + slot.tile) * a.topk;
    const int nw = L::bitmap_words(gk.nT);
    len = build_union<SAME>(a, row_a, slot.has_b, bitmaps, bitmaps + nw, unions);
    if (lane == 0) *union_len = len;
  }
  if (PAIR && !slot.has_b) {
    // no tile B (odd tile count): rows 64-127 are computed from zeros
    for (int sl = 0; sl < L::kSlabs; ++sl) {
      uint4* q4 = reinterpret_cast<uint4*>(sp + L::kQ + sl * L::kSlabBytes + 64 * 128);
      for (int e = threadIdx.x; e < 64 * 128 / 16; e += kAttnThreads) q4[e] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == kWarpPV) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kWarpK && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The softmax warps alone read the sub-block table: the producers and
  // issuers start at once, and the softmax warps meet warp 0 at named
  // barrier 2 once it has written the table.
  if (warp == 0) build_sub_desc<MODE, SAME>(a, tile_tab, unions, PAIR ? *union_len : a.topk, sub_desc);

  if (warp >= 8) setmaxnreg_dec<RegSplit<MODE>::kProducer>();
  if (warp == kWarpK || warp == kWarpV) {
    // ====================================================== TMA producers
    // Warp 8: K(j) into stage j & 1 once S(j-2) has released it;
    // warp 9: V(j) once PV(j-2) has.  Separate streams, so a K load never
    // waits behind a V release.
    if (lane == 0) {
      const bool is_k = warp == kWarpK;
      bool ok = true;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      const uint32_t buf0 = is_k ? sK : sV;
      const int full = is_k ? BAR_K_FULL : BAR_V_FULL;
      const int empty = is_k ? BAR_K_EMPTY : BAR_V_EMPTY;
      KvSeq<MODE, SAME> sq;
      sq.init(tile_tab, unions, PAIR ? *union_len : a.topk);
      const int n = sq.count(a);
      int issued = 0;
      for (int j = 0; j < n && ok; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(bar(empty + st), ((j - 2) >> 1) & 1, abort_flag, a.err)) {
          ok = false;
          break;
        }
        issued = j + 1;
        mbar_arrive_expect_tx(bar(full + st), static_cast<uint32_t>(P * L::kSlabs) * box_bytes);
#pragma unroll
        for (int p = 0; p < P; ++p) {
          const Piece pc = sq.piece(a, p);
          const TileCoord c = table_coord(tile_tab, pc.j);
          const BoxCoord bc =
              box_coord_l<BNHD>(gk, slot.bh, c.bt * gk.tt + pc.toff, c.by * gk.th, c.bx * gk.tw);
          for (int sl = 0; sl < L::kSlabs; ++sl)
            tma_load_5d(buf0 + st * L::kBufBytes + sl * L::kSlabBytes + p * box_bytes, tm, bar(full + st),
                        sl * 64, bc.c1, bc.c2, bc.c3, bc.c4);
        }
        sq.advance(a);
      }
      // Let every issued copy land before the CTA can exit (returns at once
      // when the consumers already saw these phases complete).
      for (int j = max(0, issued - 2); j < issued; ++j) mbar_wait(bar(full + (j & 1)), (j >> 1) & 1, nullptr, a.err);
    }
    __syncwarp();
  } else if (warp == kWarpPV || warp == kWarpS) {
    // ====================================================== MMA issuers
    // Warp 11: S(j) once K(j) is in and PV(j-3) has released buffer j % 3;
    // warp 10: PV(it) once P(it) and V(it) are in.  One elected lane issues
    // each group and its commits (a commit tracks the MMAs of the thread that
    // issued them; the warp is converged at every election, so it is always
    // the same lane).  Each waits on a barrier only for phases that cannot
    // complete twice before it looks (the next phase needs its own MMAs).
    constexpr uint32_t idS = idesc_f16kind_f32(kSlotRows, kSubRows, false, F16);
    constexpr uint32_t idPV = idesc_f16kind_f32(kSlotRows, D, true, F16);
    KvSeq<MODE, SAME> sq;
    sq.init(tile_tab, unions, PAIR ? *union_len : a.topk);
    const int n = sq.count(a);
    bool ok = true;
    if (warp == kWarpS) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_Q_FULL), 0, abort_flag, a.err));
      for (int j = 0; j < n && ok; ++j) {
        const int b = j % kSBufs;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_K_FULL + (j & 1)), (j >> 1) & 1, abort_flag, a.err) &&
                                         (j < kSBufs || mbar_wait(bar(BAR_S_FREE + b), ((j - kSBufs) / kSBufs) & 1,
                                                                  abort_flag, a.err)));
        if (!ok) break;
        tc_fence_after();
        if (elect_one_sync()) {
          const uint32_t tD = tmem + 128u * static_cast<uint32_t>(b);
          const uint32_t kb = sK + static_cast<uint32_t>((j & 1) * L::kBufBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int sl = kk / 4, koff = (kk % 4) * 32;    // 16 channels = 32 B within a 64-channel slab
            mma_ss(tD, smem_desc_sw128(sQ + sl * L::kSlabBytes + koff, 16, 1024),
                   smem_desc_sw128(kb + sl * L::kSlabBytes + koff, 16, 1024), idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(BAR_S_FULL + b));
          mma_commit(bar(BAR_K_EMPTY + (j & 1)));
        }
        __syncwarp();
      }
    } else {
      for (int it = 0; it < n && ok; ++it) {
        const int b = it % kSBufs;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(BAR_P_FULL + b), (it / kSBufs) & 1, abort_flag, a.err) &&
                                         mbar_wait(bar(BAR_V_FULL + (it & 1)), (it >> 1) & 1, abort_flag, a.err));
        if (!ok) break;
        tc_fence_after();
        if (elect_one_sync()) {
          const uint32_t tP = tmem + 128u * static_cast<uint32_t>(b), tO = tmem + kTmemO;
          const uint32_t vb = sV + static_cast<uint32_t>((it & 1) * L::kBufBytes);
#pragma unroll
          for (int kk = 0; kk < kSubRows / 16; ++kk)       // 16 keys = 16 rows of 128 B
            mma_ts(tO, tP + 8u * kk, smem_desc_sw128(vb + kk * 2048, L::kSlabBytes, 1024), idPV,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(BAR_PV_DONE + (it & 1)));
          mma_commit(bar(BAR_V_EMPTY + (it & 1)));
          mma_commit(bar(BAR_S_FREE + b));
          if (it == n - 1) mma_commit(bar(BAR_O_FULL));
        }
        __syncwarp();
      }
    }
    // Drain: every MMA of both issuers has finished before TMEM is freed.
    if (elect_one_sync()) mma_commit(bar(BAR_DRAIN));
    __syncwarp();
    mbar_wait(bar(BAR_DRAIN), 0, nullptr, a.err);
  } else if (warp < 8) {
    // ====================================================== softmax
    named_bar_sync(2, 256);                           // the sub-block table is written
    setmaxnreg_inc<RegSplit<MODE>::kSoftmax>();
    const int wg = warp / 4;                          // takes the sub-blocks it with it % 2 == wg
    const int r = threadIdx.x % 128;                  // query row = TMEM lane
    const bool in_b = PAIR && r >= 64;                // MODE_PAIR: rows 64-127 belong to tile B
    const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tO = tmem + lane_base + kTmemO;
    const int lg_yx = g.lg_th + g.lg_tw;
    const int lg_yx_k = gk.lg_th + gk.lg_tw;
    float* m_set = reinterpret_cast<float*>(sp + L::kRows);          // [2][128] settled max by sub-block parity
    float* fin = m_set + 2 * 128;                                     // [2][2][128] final (l, m) per warpgroup

    // which token this row is (if any)
    bool row_valid;
    int tok_t, tok_y, tok_x;
    {
      const int rr = PAIR ? (r & 63) : r;
      const int lt = rr >> lg_yx, ly = (rr >> g.lg_tw) & (g.th - 1), lx = rr & (g.tw - 1);
      tok_t = (in_b ? slot.tb0 : slot.t0) + lt;
      tok_y = (in_b ? slot.yb0 : slot.y0) + ly;
      tok_x = (in_b ? slot.xb0 : slot.x0) + lx;
      row_valid = rr < box_rows && tok_t < g.T && tok_y < g.Hh && tok_x < g.W &&
                  lt < (SHARED ? a.box_tq : g.tt) && (!in_b || slot.has_b);
    }

    int n;
    {
      KvSeq<MODE, SAME> sq;
      sq.init(tile_tab, unions, PAIR ? *union_len : a.topk);
      n = sq.count(a);
    }
    // m_own: the reference max as of this warpgroup's last sub-block (log2
    // units, scaled); l_own: its share of the row sum, relative to m_own
    float m_own = -INFINITY, l_own = 0.f;
    bool ok = true;
    const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
    for (int it = wg; it < n; it += 2) {
      // Which key columns count for this warp's rows: columns [0, 64) are
      // piece 0 and [64, 128) piece 1 (one 128-column piece outside
      // MODE_PAIR).  use0/use1: the piece was kept by this row's query tile
      // (warp-uniform); a piece that is not used contributes P = 0 without
      // any exponential.  Partial tiles at the grid edge need a column mask.
      uint32_t mw[4] = {~0u, ~0u, ~0u, ~0u};
      const uint2 dsc = sub_desc[it];
      const uint32_t fl = dsc.x >> 24;
      const bool use0 = (fl & (in_b ? 2u : 1u)) != 0;
      const bool use1 = PAIR ? (fl & (in_b ? 8u : 4u)) != 0 : use0;
      const bool geo_full = (!use0 || (fl & 16u)) && (!use1 || (fl & (PAIR ? 32u : 16u)));
      if (!geo_full) {
        const int vt0 = dsc.x & 0xff, vy0 = (dsc.x >> 8) & 0xff, vx0 = (dsc.x >> 16) & 0xff;
        const int vt1 = dsc.y & 0xff, vy1 = (dsc.y >> 8) & 0xff, vx1 = (dsc.y >> 16) & 0xff;
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

      const int b = it % kSBufs;
      const uint32_t tS = tmem + lane_base + 128u * static_cast<uint32_t>(b);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(BAR_S_FULL + b), (it / kSBufs) & 1, abort_flag, a.err))) {
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

      // Provisional reference: the one this warpgroup last settled, moved to
      // this sub-block's max if that is more than 2^8 above it (lazy
      // rescaling).  A row with no valid key so far keeps -inf, with 0 used
      // in the exponent (every P of such a row is 0).
      const float m_prov = (mx_s > m_own + kRescaleLog2) ? mx_s : m_own;
      const float mp_use = (m_prov == -INFINITY) ? 0.f : m_prov;
      // P = 2^(scale*log2(e)*S - m) on pairs of columns; row sum in 4 packed chains
      const uint64_t nm2 = f2_pack(-mp_use, -mp_use);
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
          s[c] = pack_elem2<F16>(p0, p1);
        }
        // store each half of P as soon as it is packed: the first store
        // overlaps the second half's exponentials
        tmem_st32(tS + 32u * hf, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * hf]));
      }
      float s_sum;
      {
        float a0, a1;
        f2_unpack(f2_add(f2_add(ls2[0], ls2[1]), f2_add(ls2[2], ls2[3])), a0, a1);
        s_sum = a0 + a1;
      }

      // Settle the reference in sub-block order: the one of sub-block it-1
      // (the other warpgroup's) from shared memory, moved to this block's max
      // if that is more than 2^8 above it.
      float m_prev = -INFINITY;
      if (it > 0) {
        const int ip = it - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(BAR_M_READY + (ip & 1)), (ip >> 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        m_prev = m_set[(ip & 1) * 128 + r];
      }
      const float m_it = (mx_s > m_prev + kRescaleLog2) ? mx_s : m_prev;
      const float mi_use = (m_it == -INFINITY) ? 0.f : m_it;
      // P went out against m_prov: when the other warpgroup moved the
      // reference meanwhile (rare), scale the stored P (and its sum) to m_it
      const float f_p = (m_prov == m_it || m_prov == -INFINITY) ? 1.f : ex2_approx(mp_use - mi_use);
      if (__any_sync(0xffffffffu, f_p != 1.f)) {
        tmem_wait_st();
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t pv[32];
          tmem_ld32(tS + 32u * h2, pv);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float2 f = unpack_elem2<F16>(pv[c]);
            pv[c] = pack_elem2<F16>(f.x * f_p, f.y * f_p);
          }
          tmem_st32(tS + 32u * h2, pv);
        }
      }
      {
        const float mo_use = (m_own == -INFINITY) ? 0.f : m_own;
        l_own = (m_own == m_it ? l_own : l_own * ex2_approx(mo_use - mi_use)) + s_sum * f_p;
        m_own = m_it;
      }
      // O holds PV(0 .. it-1), relative to m_prev.  When this sub-block moved
      // the reference (rare), O is rescaled after PV(it-1) has completed and
      // before P_FULL lets PV(it) start; otherwise P_FULL goes first.  The
      // PV_DONE phase of it-1 is waited here either way, and M_READY follows
      // it: the barrier's next phase of that parity (PV(it+1)) needs the
      // other warpgroup's P after this M_READY, so no phase is missed.
      const bool o_fix = it > 0 && __any_sync(0xffffffffu, m_it != m_prev);
      bool pv_seen = it == 0;
      if (o_fix) {
        const int ip = it - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(BAR_PV_DONE + (ip & 1)), (ip >> 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        pv_seen = true;
        tc_fence_after();
        const float f_o = (m_it == m_prev) ? 1.f : ((m_prev == -INFINITY) ? 0.f : ex2_approx(m_prev - m_it));
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t ov[32];
          tmem_ld32(tO + 32u * c4, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f_o);
          tmem_st32(tO + 32u * c4, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BAR_P_FULL + b));
      if (!pv_seen) {
        const int ip = it - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(BAR_PV_DONE + (ip & 1)), (ip >> 1) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
      }
      m_set[(it & 1) * 128 + r] = m_it;
      mbar_arrive(bar(BAR_M_READY + (it & 1)));
    }

    // ---- epilogue: the row sum from both warpgroups' shares, then each
    // warpgroup writes half of O's columns: O / l -> the input type; LSE
    fin[(wg * 2 + 0) * 128 + r] = l_own;
    fin[(wg * 2 + 1) * 128 + r] = m_own;
    named_bar_sync(1, 256);                           // both softmax warpgroups, once each
    const float l_o = fin[((1 - wg) * 2 + 0) * 128 + r], m_o = fin[((1 - wg) * 2 + 1) * 128 + r];
    const float m_fin = fmaxf(m_own, m_o);
    const float mf_use = (m_fin == -INFINITY) ? 0.f : m_fin;
    const float l_tot = (m_own == -INFINITY ? 0.f : l_own * ex2_approx((m_own) - mf_use)) +
                        (m_o == -INFINITY ? 0.f : l_o * ex2_approx(m_o - mf_use));
    // O leaves through the Q buffer (every MMA that read Q has completed by
    // O_FULL), in the layout the Q boxes were loaded with (128-byte swizzle:
    // 16-byte chunk c of row r sits at chunk c ^ (r % 8)), then one TMA store
    // per box and slab writes whole lines and drops the rows outside the grid.
    bool staged = false;
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar(BAR_O_FULL), 0, abort_flag, a.err))) {
      tc_fence_after();
      const float inv_l = 1.f / l_tot;
      const size_t N = static_cast<size_t>(g.T) * g.Hh * g.W;
      const size_t n_tok = (static_cast<size_t>(tok_t) * g.Hh + tok_y) * g.W + tok_x;
      const uint32_t orow_s = sQ + static_cast<uint32_t>(r) * 128u;
#pragma unroll
      for (int c4 = wg * (D / 64); c4 < (wg + 1) * (D / 64); ++c4) {
        uint32_t ov[32];
        tmem_ld32(tO + 32u * c4, ov);
        tmem_wait_ld();
        if (row_valid) {
          float of[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) of[e] = __uint_as_float(ov[e]) * inv_l;
          if (a.gate != nullptr) {
            // pooled coarse branch: O += gate * o_coarse of this row's query tile
            const uint4* gp = reinterpret_cast<const uint4*>(a.gate + token_offset(g, slot.bh, n_tok) + 32 * c4);
            const float4* cp = reinterpret_cast<const float4*>(
                a.coarse + (static_cast<size_t>(slot.bh) * g.nT + slot.tile + (in_b ? 1 : 0)) * D + 32 * c4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint4 gv = __ldg(gp + e);
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
              const float4 c0 = __ldg(cp + 2 * e), c1 = __ldg(cp + 2 * e + 1);
              const float cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 gf = unpack_elem2<F16>(gw[u]);
                of[8 * e + 2 * u] = fmaf(gf.x, cw[2 * u], of[8 * e + 2 * u]);
                of[8 * e + 2 * u + 1] = fmaf(gf.y, cw[2 * u + 1], of[8 * e + 2 * u + 1]);
              }
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_elem2<F16>(of[2 * e], of[2 * e + 1]);
          const uint32_t slab_row = orow_s + static_cast<uint32_t>(c4 >> 1) * L::kSlabBytes;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            st_shared_v4(slab_row + static_cast<uint32_t>(((c4 & 1) * 4 + e) ^ (r & 7)) * 16u, pk[4 * e],
                         pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      fence_proxy_async_smem();
      staged = true;
      if (row_valid && wg == 0)
        __stcs(a.lse + static_cast<size_t>(slot.bh) * N + n_tok, (m_fin + log2f(l_tot)) * 0.69314718055994530942f);
    }
    named_bar_sync(1, 256);                           // O staged by both warpgroups
    if (threadIdx.x == 0 && staged) {
      const int b = slot.bh / g.H, h = slot.bh - b * g.H;
      for (int sl = 0; sl < L::kSlabs; ++sl) {
        // [B, N, H, d]: channel coordinate h * d + slab, batch last (the O
        // map's dimensions); [B, H, N, d]: as the Q map
        const int c0 = BNHD ? h * D + sl * 64 : sl * 64, c4 = BNHD ? b : slot.bh;
        const uint32_t src = sQ + static_cast<uint32_t>(sl * L::kSlabBytes);
        tma_store_5d(&tmO, src, c0, slot.x0, slot.y0, slot.t0, c4);
        if (PAIR && slot.has_b) tma_store_5d(&tmO, src + box_bytes, c0, slot.xb0, slot.yb0, slot.tb0, c4);
      }
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpPV) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace vsa
