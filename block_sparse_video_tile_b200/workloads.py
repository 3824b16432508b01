"""The workloads this library is measured and checked on.

Each entry is a latent-grid attention problem: batch B, heads H, head_dim d,
post-patch latent grid (T, Hh, W), spatio-temporal tile (tt, th, tw), and the
number of key/value tiles kept per query tile (topk).

* ``tiny``     -- 8x8x8 grid, 4x4x4 tiles (8 tiles), 2 heads of 64: small
  enough for the pure-Python oracle.
* ``wan5b``    -- the FastWan2.2-TI2V-5B shape from the FastVideo VSA user guide
  ("Wan top-k behavior"): grid (31, 22, 40) = 27280 tokens, 4x8x8 tiles ->
  120 tiles, topk 64 (keep ratio 53.3%); 24 heads of 128.
* ``wan14b``   -- the Wan2.1-T2V-14B 768x1280x69-frame shape from the Sliding
  Tile Attention page's example run: grid (18, 48, 80), 4x8x8 -> 300 tiles,
  topk 30; 40 heads of 128; structured Q/K.
* ``longcat``  -- a LongCat-Video-like 720p grid (12, 48, 80), 4x4x4 chunks ->
  720 tiles, sparsity 0.9375 (topk 45) as in the fastbsa page's "Use" example;
  32 heads of 128; structured Q/K.
* ``longcat_kv`` -- the LongCat-like grid called the fastbsa way: [B, N, H, d]
  tensors, keys and values over 16 frames (4 conditioning frames more than the
  queries' 12), sparsity 0.9375 -> 60 of 960 key tiles.
* ``sweep``    -- the Wan-5B shape at topk 8, 16, 32, 64 and 120 (120 = all
  tiles, which must equal dense attention), N(0, 1) and structured inputs.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid: tuple
    d: int
    tile: tuple
    topk: int
    kind: str = "normal"
    dtype: str = "bf16"        # element type of Q, K, V, O: "bf16" or "f16"
    layout: str = "bhnd"       # "bhnd" = [B, H, N, d] or "bnhd" = [B, N, H, d]
    grid_k: tuple | None = None   # key/value grid (None: the query grid)
    tile_k: tuple | None = None   # key/value tile (None: the query tile)
    prefix_tiles: int = 0         # key/value tiles kept for every query tile

    @property
    def N(self) -> int:
        T, Hh, W = self.grid
        return T * Hh * W

    @property
    def kv_grid(self) -> tuple:
        return self.grid if self.grid_k is None else self.grid_k

    @property
    def kv_tile(self) -> tuple:
        return self.tile if self.tile_k is None else self.tile_k

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny", 1, 2, (8, 8, 8), 64, (4, 4, 4), 2)
WAN5B = Workload("wan5b", 1, 24, (31, 22, 40), 128, (4, 8, 8), 64)
WAN14B = Workload("wan14b", 1, 40, (18, 48, 80), 128, (4, 8, 8), 30, "field")
LONGCAT = Workload("longcat", 1, 32, (12, 48, 80), 128, (4, 4, 4), 45, "field")
# The LongCat-style call of the fastbsa page ("Use"): [B, N, H, d] tensors, keys and
# values over 4 more latent frames than the queries (conditioning frames), 4x4x4
# chunks on both sides, sparsity 0.9375 -> 60 of 960 key/value tiles kept.
LONGCAT_KV = Workload("longcat_kv", 1, 32, (12, 48, 80), 128, (4, 4, 4), 60, "field", layout="bnhd",
                      grid_k=(16, 48, 80))
SWEEP_TOPK = (8, 16, 32, 64, 120)
SWEEP = tuple(WAN5B.with_(name=f"sweep_k{k}_{kind}", topk=k, kind=kind)
              for kind in ("normal", "field") for k in SWEEP_TOPK)

ALL = {w.name: w for w in (TINY, WAN5B, WAN14B, LONGCAT, LONGCAT_KV) + SWEEP}
