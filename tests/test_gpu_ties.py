"""Exact ties in tile selection, on the GPU against the oracle.

Every key tile copies one of P token patterns (a grid of full tiles), so the
pooled key means repeat exactly: on the GPU every score of a row falls into
P groups of bit-identical values (the same sums in the same order).  Ties must
go to the lower tile index (FastVideo VSA user guide, "Wan top-k behavior":
top-k key/value blocks per query block; the lower-index rule is this
library's reading), so the GPU's indices must equal the oracle's top-k of the
tied scores exactly.  The oracle's float64 matrix product can round equal
columns one ulp apart, so the reference ties them explicitly: tile j takes
the oracle's score of tile j % P (a tile of the same pattern).

The cases reach each way the top-k settles its threshold: a tied group of
exactly the missing size (P = 16: 45 equal keys for topk 45), a tied group
gathered into registers (P = 8: 90 equal keys), a tied group too large to
gather (P = 4: 180 equal keys), and, at a narrow-kernel size, a tie straddling
the threshold (10 equal keys per group, topk 12).
"""
import numpy as np
import pytest
import torch

from block_sparse_video_tile_b200 import api, synth
from oracle import vsa_oracle as vo

CASES = [
    # grid, tile, patterns, topk
    ((12, 48, 80), (4, 4, 4), 16, 45),
    ((12, 48, 80), (4, 4, 4), 8, 45),
    ((12, 48, 80), (4, 4, 4), 4, 45),
    ((8, 32, 40), (4, 8, 8), 4, 12),
]


def _tile_periodic_keys(grid, tile, P, d, rng):
    """[1, 1, N, d] bf16 bits: token (t, y, x) of tile j takes row (t%tt, y%th,
    x%tw) of pattern j % P (full tiles only)."""
    T, Hh, W = grid
    tt, th, tw = tile
    assert T % tt == 0 and Hh % th == 0 and W % tw == 0
    vol = tt * th * tw
    pats = synth.f32_to_bf16_bits(rng.standard_normal((P, vol, d), dtype=np.float32))
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(W), indexing="ij")
    j = ((t // tt) * (Hh // th) + (y // th)) * (W // tw) + (x // tw)
    pos = ((t % tt) * th + (y % th)) * tw + (x % tw)
    return pats[(j % P).reshape(-1), pos.reshape(-1)][None, None]


@pytest.mark.gpu
@pytest.mark.parametrize("grid,tile,P,topk", CASES, ids=[f"P{c[2]}_k{c[3]}_{c[1][1]}" for c in CASES])
def test_exact_ties_go_to_lower_index(grid, tile, P, topk):
    rng = np.random.default_rng(11)
    d = 128
    N = grid[0] * grid[1] * grid[2]
    q = synth.f32_to_bf16_bits(rng.standard_normal((1, 1, N, d), dtype=np.float32))
    k = _tile_periodic_keys(grid, tile, P, d, rng)
    qd, kd = (torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).cuda() for x in (q, k))
    idx = api.select(qd, kd, grid, tile, topk)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    _, scores, _ = vo.select(q, k, grid, tile, topk)
    nT = scores.shape[-1]
    tied = scores[0, 0][:, np.arange(nT) % P]
    gpu = idx.cpu().numpy()[0, 0]
    exact = 0
    for i in range(tied.shape[0]):
        gap, _ = vo.tie_gap(tied[i], topk)
        if gap == 0.0 or gap >= 1e-5:
            # the cut falls inside a tied group, or clearly between two groups
            assert np.array_equal(gpu[i], vo.topk_row(tied[i], topk)), f"row {i}: tie resolution differs"
            exact += 1
        else:
            # two groups within float32 rounding of each other at the cut
            assert vo.selection_is_valid(gpu[i], tied[i], topk), f"row {i}: invalid selection"
    assert exact >= 0.95 * tied.shape[0]
