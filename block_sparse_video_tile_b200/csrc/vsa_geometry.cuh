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
};

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
