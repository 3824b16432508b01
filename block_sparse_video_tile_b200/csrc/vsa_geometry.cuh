// vsa_geometry.cuh -- the 3-D tile index map, evaluated inside the kernels.
//
// FastVideo VSA user guide ("Wan top-k behavior"): the post-patch latent grid
// (T, Hh, W) is cut into (tt, th, tw) blocks with ceil division per axis, so
// edge blocks are partial; grid (31, 22, 40) with 4x8x8 blocks gives 120.
// fastbsa page ("How it works"): the token <-> block map is evaluated in the
// kernel instead of permuting Q/K/V into block order through HBM.
//
// Token n of a head is (t, y, x) with n = (t * Hh + y) * W + x.  Tile j is
// (bt, by, bx) with j = (bt * nTy + by) * nTx + bx.  Inside a tile, local row
// r = (lt * th + ly) * tw + lx (raster order, the order a TMA box writes).
#pragma once

#include <cstdint>

namespace vsa {

struct Geom {
  int B, H, T, Hh, W, d;
  int tt, th, tw;
  int nTt, nTy, nTx, nT;  // tiles per axis and in total
  int lg_tt, lg_th, lg_tw;  // log2 of the (power-of-two) tile extents
  int vol;                  // tt * th * tw
  int f16;                  // element type: 0 bfloat16, 1 float16
  int layout;               // 0: [B, H, N, d]; 1: [B, N, H, d]
  int prefix;               // key/value side: tiles 0 .. prefix-1 are always kept (0 on the query side)
};

// A query-side and a key/value-side Geom share B, H, d, f16 and layout; each
// has its own grid, tile and tile count.

// TMA coordinates (after the channel coordinate) of the box whose first token
// is (t, y, x) of head bh.  The [B, H, N, d] view is (d, W, Hh, T, B*H); the
// [B, N, H, d] view is (d, H, W, Hh, B*T) -- batch and time fold into one
// dimension because a batch's stride is T times a frame's.
struct BoxCoord {
  int c1, c2, c3, c4;
};

__host__ __device__ inline BoxCoord box_coord(const Geom& g, int bh, int t, int y, int x) {
  BoxCoord c;
  if (g.layout == 1) {
    const int b = bh / g.H;
    c.c1 = bh - b * g.H;
    c.c2 = x;
    c.c3 = y;
    c.c4 = b * g.T + t;
  } else {
    c.c1 = x;
    c.c2 = y;
    c.c3 = t;
    c.c4 = bh;
  }
  return c;
}

// The same with the layout fixed at compile time (kernels instantiated per
// layout: no division or branch in their box-issuing loops).
template <bool BNHD>
__host__ __device__ inline BoxCoord box_coord_l(const Geom& g, int bh, int t, int y, int x) {
  BoxCoord c;
  if (BNHD) {
    const int b = bh / g.H;
    c.c1 = bh - b * g.H;
    c.c2 = x;
    c.c3 = y;
    c.c4 = b * g.T + t;
  } else {
    c.c1 = x;
    c.c2 = y;
    c.c3 = t;
    c.c4 = bh;
  }
  return c;
}

// Element offset of token n of head bh (N = T * Hh * W tokens per head).
__host__ __device__ inline size_t token_offset(const Geom& g, int bh, size_t n) {
  const size_t N = static_cast<size_t>(g.T) * g.Hh * g.W;
  if (g.layout == 1) {
    const int b = bh / g.H;
    return ((static_cast<size_t>(b) * N + n) * g.H + (bh - b * g.H)) * g.d;
  }
  return (static_cast<size_t>(bh) * N + n) * g.d;
}

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ inline int ilog2_exact(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return ((1 << l) == v) ? l : -1;
}

// Tile coordinates of tile j.
struct TileCoord {
  int bt, by, bx;
};

__host__ __device__ inline TileCoord tile_coord(const Geom& g, int j) {
  TileCoord c;
  c.bx = j % g.nTx;
  c.by = (j / g.nTx) % g.nTy;
  c.bt = j / (g.nTx * g.nTy);
  return c;
}

// Valid extents of tile (bt, by, bx) along each axis (partial at the edges).
__host__ __device__ inline void tile_extent(const Geom& g, const TileCoord& c, int& vt, int& vy,
                                            int& vx) {
  vt = min(g.tt, g.T - c.bt * g.tt);
  vy = min(g.th, g.Hh - c.by * g.th);
  vx = min(g.tw, g.W - c.bx * g.tw);
}

}  // namespace vsa
