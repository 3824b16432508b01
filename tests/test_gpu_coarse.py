"""Pooled coarse branch on the GPU against the float64 oracle, through the C ABI.

The branch (FastVideo VSA user guide, "Checkpoint behavior": a learned
gate_compress compensation added to the sparse branch) has no formula on the
pages; the oracle's reading -- tile-level attention over the tiles' mean
rows, added to each query tile's tokens through a gate -- is pinned in
tests/test_oracle_pins.py.  Here vsa_select_coarse and vsa_attn_fwd_gated
are checked against it: the tile selection is unchanged, o_coarse matches the
oracle's to float32 accuracy, the gated output is within the O tolerances of
the oracle's sparse output plus gate * o_coarse, and a zero gate leaves O
bit-identical to vsa_attn_fwd.
"""
import numpy as np
import pytest
import torch

from block_sparse_video_tile_b200 import api, synth
from block_sparse_video_tile_b200.workloads import LONGCAT, TINY, WAN5B, Workload
from oracle import vsa_oracle as vo
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

COARSE_ABS = 1e-4        # o_coarse: float32 means, scores and softmax against float64

CASES = [
    TINY,
    Workload("ragged256", 1, 2, (9, 20, 20), 128, (4, 8, 8), 5),
    Workload("ragged64_d64", 1, 3, (5, 9, 11), 64, (4, 4, 4), 6),
    Workload("vol128", 2, 1, (6, 12, 20), 128, (2, 8, 8), 4),
    Workload("pair_odd", 1, 3, (4, 4, 20), 128, (4, 4, 4), 3),
    Workload("kv_tile_shared", 1, 2, (9, 20, 20), 128, (4, 8, 8), 6, "field", grid_k=(10, 18, 30),
             tile_k=(2, 8, 16)),
    Workload("bnhd_pair_f16", 2, 2, (6, 10, 14), 128, (4, 4, 4), 5, "field", layout="bnhd", dtype="f16"),
]


def _gate(w, seed):
    """A gate tensor in the workload's layout and type, and its float64 values [B, H, N, d]."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((w.B, w.H, w.N, w.d)).astype(np.float32)
    bits = synth.f32_to_f16_bits(g) if w.dtype == "f16" else synth.f32_to_bf16_bits(g)
    dev = gu.to_dev(bits, w.dtype)
    if w.layout == "bnhd":
        dev = dev.permute(0, 2, 1, 3).contiguous()
    return dev, vo.widen(bits, w.dtype)


def _check(w, seed, heads=None, tiles_per_head=None):
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=seed)
    scale = w.d ** -0.5
    idx, coarse = api.select_coarse(qd, kd, vd, w.grid, w.tile, w.topk, scale=scale, **gu.sel(w))
    idx_plain = api.select(qd, kd, w.grid, w.tile, w.topk, **gu.sel(w))
    torch.cuda.synchronize()
    gu.assert_no_device_error()
    assert torch.equal(idx, idx_plain), "the coarse select changed the tile selection"
    gate_d, gate = _gate(w, seed + 100)
    o_g, lse_g = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile, scale=scale, coarse=coarse, gate=gate_d, **gu.geo(w))
    o_p, lse_p = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile, scale=scale, **gu.geo(w))
    zero = torch.zeros_like(gate_d)
    o_z, lse_z = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile, scale=scale, coarse=coarse, gate=zero, **gu.geo(w))
    gu.assert_no_device_error()
    assert torch.equal(o_z.view(torch.int16), o_p.view(torch.int16)), "a zero gate changed O"
    assert torch.equal(lse_g, lse_p) and torch.equal(lse_z, lse_p)
    gi = idx.cpu().numpy()
    cg = coarse.cpu().numpy()
    og = gu.to_bhnd(o_g, w).float().cpu().numpy()
    toks = vo.tile_tokens(w.grid, w.tile)
    heads = heads if heads is not None else range(w.B * w.H)
    errs, max_c = [], 0.0
    for bh in heads:
        b, h = divmod(bh, w.H)
        Q, K, V = (vo.widen(x[b, h], w.dtype) for x in (q, k, v))
        oc = vo.coarse_head(Q, K, V, w.grid, w.tile, scale, grid_k=w.kv_grid, tile_k=w.kv_tile)
        max_c = max(max_c, float(np.abs(cg[b, h] - oc).max()))
        ts = list(range(len(toks))) if tiles_per_head is None else tiles_per_head
        O, _ = vo.attend_head(Q, K, V, w.grid, w.tile, gi[b, h], scale, query_tiles=ts, grid_k=w.kv_grid,
                              tile_k=w.kv_tile)
        rows = np.concatenate([toks[i] for i in ts])
        ref = vo.gated_output(np.nan_to_num(O), gate[b, h], oc, w.grid, w.tile)
        errs.append(np.abs(og[b, h][rows] - ref[rows]).reshape(-1))
    assert max_c <= COARSE_ABS, f"o_coarse max-abs {max_c}"
    e = np.concatenate(errs)
    assert e.max() <= gu.O_MAX_ABS and e.mean() <= gu.O_MEAN_ABS, (e.max(), e.mean())
    return max_c, float(e.max()), float(e.mean())


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_coarse_small(w):
    print(w.name, _check(w, seed=0))


@pytest.mark.parametrize("w", [WAN5B, LONGCAT], ids=lambda w: w.name)
def test_coarse_full_size(w):
    """Full-size workloads: o_coarse of two whole heads, gated O on sampled query tiles."""
    nT = vo.num_tiles(w.grid, w.tile)
    print(w.name, _check(w, seed=0, heads=[0, w.B * w.H - 1], tiles_per_head=[0, 1, nT // 2, nT - 1]))


def test_gated_requires_both():
    w = CASES[1]
    _, (qd, kd, vd) = gu.inputs(w, seed=0)
    idx, coarse = api.select_coarse(qd, kd, vd, w.grid, w.tile, w.topk)
    with pytest.raises(ValueError):
        api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile, coarse=coarse)
