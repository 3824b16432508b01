"""CUDA path vs the float64 oracle, through the C ABI.

Small cases are compared element by element on every token; they span
several tiles and ragged (partial) edge tiles on every axis, both tile
volumes (64 and 256 tokens, plus 128), both head sizes and batch > 1.  The
five full-size workloads run in the configuration the benchmark times and are
checked on every selected index and on every query tile of two whole heads
(edge tiles included) of the attention output.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_video_tile_b200 import api
from block_sparse_video_tile_b200.workloads import ALL, LONGCAT, SWEEP, TINY, WAN14B, WAN5B, Workload
from oracle import vsa_oracle as vo
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

SMALL = [
    TINY,
    TINY.with_(name="tiny_s1"),
    Workload("ragged256", 1, 2, (9, 20, 20), 128, (4, 8, 8), 5),
    Workload("ragged256_d64", 2, 1, (9, 20, 20), 64, (4, 8, 8), 7),
    Workload("ragged256_field", 1, 2, (10, 17, 24), 128, (4, 8, 8), 4, "field"),
    Workload("ragged64", 1, 2, (6, 10, 14), 128, (4, 4, 4), 5),
    Workload("ragged64_d64", 1, 3, (5, 9, 11), 64, (4, 4, 4), 6),
    Workload("vol128", 2, 1, (6, 12, 20), 128, (2, 8, 8), 4),
    # 128-token tiles, an odd count of (head, tile) units (3 heads x 9 tiles):
    # the last CTA's second slot is empty and its MMA issuer runs alone
    Workload("tile_odd", 1, 3, (6, 8, 24), 128, (2, 8, 8), 4),
    Workload("topk1", 1, 2, (9, 20, 20), 128, (4, 8, 8), 1),
    # 64-token tiles, odd tile count per head: the last pair has no tile B
    Workload("pair_odd", 1, 3, (4, 4, 20), 128, (4, 4, 4), 3),
    # 64-token tiles with structured inputs: neighbouring tiles share kept tiles
    Workload("pair_field", 1, 2, (8, 12, 20), 128, (4, 4, 4), 7, "field"),
    # 256-token tiles split along t with tt = 2 and with tt = 8
    Workload("shared_tt2", 1, 2, (7, 16, 24), 128, (2, 8, 16), 5),
    Workload("shared_tt8", 1, 2, (13, 8, 12), 64, (8, 4, 8), 4),
    # float16 inputs (the Wan route takes FP16 or BF16) in each kernel mode
    Workload("f16_shared", 1, 2, (9, 20, 20), 128, (4, 8, 8), 5, dtype="f16"),
    Workload("f16_tile_d64", 2, 1, (6, 12, 20), 64, (2, 8, 8), 4, dtype="f16"),
    Workload("f16_pair", 1, 2, (6, 10, 14), 128, (4, 4, 4), 5, "field", dtype="f16"),
    # [B, N, H, d] layout with B = 2 and a partial last t-tile, whose boxes read
    # the next batch's first frames (masked), in each kernel mode
    Workload("bnhd_shared", 2, 2, (9, 20, 20), 128, (4, 8, 8), 5, layout="bnhd"),
    Workload("bnhd_tile", 2, 3, (6, 12, 20), 64, (4, 4, 8), 4, layout="bnhd"),
    Workload("bnhd_pair", 2, 2, (6, 10, 14), 128, (4, 4, 4), 5, "field", layout="bnhd"),
    # keys and values on their own grid (fastbsa page, "Use": latent_shape_k,
    # chunk_3d_shape_k), with the same or another tile of equal volume
    Workload("kv_grid_shared", 1, 2, (9, 20, 20), 128, (4, 8, 8), 6, grid_k=(13, 16, 24)),
    Workload("kv_tile_shared", 1, 2, (9, 20, 20), 128, (4, 8, 8), 6, "field", grid_k=(10, 18, 30),
             tile_k=(2, 8, 16)),
    Workload("kv_pair", 1, 2, (6, 10, 14), 128, (4, 4, 4), 5, "field", grid_k=(7, 12, 9), tile_k=(2, 4, 8)),
    Workload("kv_tile_bnhd", 2, 1, (6, 12, 20), 64, (2, 8, 8), 4, grid_k=(5, 9, 26), tile_k=(4, 4, 8),
             layout="bnhd"),
    # always-kept prefix tiles (user guide, "Choose top-k": H3 keeps all prefix
    # blocks, 64-token blocks): the keys' first 4 frames (12 tiles) are kept by
    # every query tile, plus 6 by score; and a self-attention case whose first
    # temporal slice of tiles is the prefix, with topk == prefix_tiles on one
    Workload("h3_prefix", 1, 2, (8, 12, 16), 128, (4, 4, 4), 18, "field", grid_k=(12, 12, 16), prefix_tiles=12),
    Workload("h3_prefix_bnhd", 2, 2, (8, 12, 16), 64, (4, 4, 4), 12, grid_k=(12, 12, 16), prefix_tiles=12,
             layout="bnhd"),
    Workload("prefix_self", 1, 2, (9, 20, 20), 128, (4, 8, 8), 12, "field", prefix_tiles=9),
    # options combined: fp16, [B, N, H, d], own key/value grid and tile, prefix tiles
    Workload("combo_f16_shared", 2, 2, (9, 20, 20), 128, (4, 8, 8), 8, "field", dtype="f16", layout="bnhd",
             grid_k=(10, 18, 30), tile_k=(2, 8, 16), prefix_tiles=4),
    Workload("combo_f16_pair", 1, 3, (6, 10, 14), 64, (4, 4, 4), 9, "field", dtype="f16", layout="bnhd",
             grid_k=(7, 12, 9), tile_k=(2, 4, 8), prefix_tiles=9),
    Workload("combo_tile_d64", 2, 2, (6, 12, 20), 64, (2, 8, 8), 5, grid_k=(5, 9, 26), tile_k=(4, 4, 8),
             prefix_tiles=2),
]
BY_NAME = {w.name: w for w in SMALL}


def _seed(w):
    return 1 if w.name == "tiny_s1" else 0


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_full_compare(w):
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=_seed(w))
    scale = w.d ** -0.5
    idx = api.select(qd, kd, w.grid, w.tile, w.topk, **gu.sel(w))
    torch.cuda.synchronize()
    gu.assert_no_device_error()
    scores = gu.oracle_scores(q, k, w)
    rows, ties = gu.check_selection(idx.cpu().numpy(), scores, w.topk)
    # attention on the GPU's own selection (so a tie row is still checked)
    o, lse = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile, scale=scale, **gu.geo(w))
    gu.assert_no_device_error()
    gu.check_attention(o, lse, q, k, v, w, idx.cpu().numpy(), scale)


@pytest.mark.parametrize("w", [BY_NAME[n] for n in ("ragged256", "ragged64", "vol128", "kv_tile_shared",
                                                     "kv_pair", "bnhd_tile")], ids=lambda w: w.name)
def test_oracle_indices_attention(w):
    """Attention alone, fed an arbitrary selection."""
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=3)
    nT, nTk = vo.num_tiles(w.grid, w.tile), vo.num_tiles(w.kv_grid, w.kv_tile)
    rng = np.random.default_rng(5)
    idx = np.sort(np.stack([[rng.choice(nTk, w.topk, replace=False) for _ in range(nT)]
                            for _ in range(w.B * w.H)]), axis=-1).reshape(w.B, w.H, nT, w.topk)
    idx = idx.astype(np.int32)
    o, lse = api.attn_fwd(qd, kd, vd, torch.from_numpy(idx).cuda(), w.grid, w.tile, scale=0.3, **gu.geo(w))
    gu.assert_no_device_error()
    gu.check_attention(o, lse, q, k, v, w, idx, 0.3)


@pytest.mark.parametrize("w", [BY_NAME[n] for n in ("ragged256", "ragged64", "ragged256_d64", "kv_grid_shared",
                                                     "kv_pair", "bnhd_shared")], ids=lambda w: w.name)
def test_all_tiles_equal_dense(w):
    """topk == num_blocks keeps every tile: the result is dense attention
    (FastVideo VSA user guide, "Wan top-k behavior"), over all Nk keys."""
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=4)
    nTk = vo.num_tiles(w.kv_grid, w.kv_tile)
    idx = api.select(qd, kd, w.grid, w.tile, nTk, **gu.geo(w))
    assert (idx.cpu().numpy() == np.arange(nTk)).all()
    scale = w.d ** -0.5
    o, lse = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile, scale=scale, **gu.geo(w))
    gu.assert_no_device_error()
    og, lg = gu.to_bhnd(o, w).float().cpu().numpy(), lse.cpu().numpy()
    for b in range(w.B):
        for h in range(w.H):
            Od, Ld = vo.dense_bruteforce(*(vo.widen(x[b, h], w.dtype) for x in (q, k, v)), scale)
            e = np.abs(og[b, h] - Od)
            assert e.max() <= gu.O_MAX_ABS and e.mean() <= gu.O_MEAN_ABS
            assert np.abs(lg[b, h] - Ld).max() <= gu.LSE_ABS


def test_deterministic():
    w = SMALL[2]
    _, (qd, kd, vd) = gu.inputs(w, seed=9)
    outs = []
    for _ in range(2):
        idx = api.select(qd, kd, w.grid, w.tile, w.topk)
        o, lse = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile)
        outs.append((idx.clone(), o.clone(), lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1].view(torch.int16), outs[1][1].view(torch.int16))
    assert torch.equal(outs[0][2], outs[1][2])


def test_out_of_range_index_reports_error():
    """An index outside [0, nT) is reported through the device error word;
    the kernel reads tile 0 in its place (every load stays in bounds)."""
    w = SMALL[2]
    _, (qd, kd, vd) = gu.inputs(w, seed=2)
    idx = api.select(qd, kd, w.grid, w.tile, w.topk)
    gu.assert_no_device_error()
    idx[0, 0, 3, -1] = 10_000                  # last entry: the list stays ascending
    o, lse = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile)
    assert api.device_error(reset=True) == 2
    assert torch.isfinite(lse).all()


@pytest.mark.parametrize("name", ["ragged256", "vol128", "ragged64"])
def test_unordered_index_reports_error(name):
    """A kept list that is not strictly ascending (a repeated tile, or two
    tiles swapped) is reported through the device error word in every kernel
    mode (256-, 128- and 64-token tiles; in the last, row 3 is tile B of a
    pair); the kernel completes and an untouched list gives no error."""
    w = BY_NAME[name]
    _, (qd, kd, vd) = gu.inputs(w, seed=2)
    idx = api.select(qd, kd, w.grid, w.tile, w.topk)
    api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile)
    gu.assert_no_device_error()
    for edit in ("repeat", "swap"):
        bad = idx.clone()
        if edit == "repeat":
            bad[0, 0, 3, 1] = bad[0, 0, 3, 0]
        else:
            bad[0, -1, 3, 0], bad[0, -1, 3, 1] = idx[0, -1, 3, 1], idx[0, -1, 3, 0]
        o, lse = api.attn_fwd(qd, kd, vd, bad, w.grid, w.tile)
        assert api.device_error(reset=True) == 3, edit
        assert torch.isfinite(lse).all()


def test_bad_topk_raises():
    w = SMALL[2]
    _, (qd, kd, vd) = gu.inputs(w)
    with pytest.raises(Exception):
        api.select(qd, kd, w.grid, w.tile, 0)
    with pytest.raises(Exception):
        api.select(qd, kd, w.grid, w.tile, 28)


# ----------------------------------------------------------- full-size workloads
FULL = [WAN5B, WAN14B, LONGCAT, WAN5B.with_(name="wan5b_f16", dtype="f16")]


def _check_heads(w):
    """(b, h, query tile) for every query tile of the first and the last head:
    whole heads, edge tiles included (the float64 oracle takes a few seconds
    per Wan-shape head)."""
    nT = vo.num_tiles(w.grid, w.tile)
    heads = sorted({0, w.B * w.H - 1})
    return [(bh // w.H, bh % w.H, i) for bh in heads for i in range(nT)]


def _full_case(w, seed=0, topks=None):
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=seed)
    scores = gu.oracle_scores(q, k, w)
    report = {}
    for topk in (topks or [w.topk]):
        idx = api.select(qd, kd, w.grid, w.tile, topk, **gu.sel(w))
        gi = idx.cpu().numpy()
        rows, ties = gu.check_selection(gi, scores, topk)
        o, lse = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile, **gu.geo(w))
        gu.assert_no_device_error()
        errs = gu.check_attention(o, lse, q, k, v, w, gi, w.d ** -0.5, tiles=_check_heads(w))
        report[topk] = (rows, ties, errs)
    return report


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size(w):
    rep = _full_case(w)
    print(w.name, rep)


# A LongCat-style call (fastbsa page, "Use"): [B, N, H, d] tensors, keys and
# values over 4 more latent frames than the queries, 4x4x4 chunks on both
# sides, sparsity 0.9375 (960 key tiles -> 60 kept); 8 of the 32 heads.
LONGCAT_KV = LONGCAT.with_(name="longcat_kv_bnhd", H=8, layout="bnhd", grid_k=(16, 48, 80), topk=60)


def test_longcat_style_call():
    w = LONGCAT_KV
    assert api.topk_from_sparsity(w.grid, w.tile, 0.9375, w.grid_k) == w.topk
    rep = _full_case(w)
    print(w.name, rep)


def test_forward_with_sparsity():
    w = BY_NAME["kv_pair"]
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=2)
    nTk = vo.num_tiles(w.kv_grid, w.kv_tile)
    topk = vo.topk_from_sparsity(nTk, 0.8)
    o, lse, idx = api.forward(qd, kd, vd, w.grid, w.tile, sparsity=0.8, **gu.geo(w))
    assert idx.shape[-1] == topk
    o2, lse2, idx2 = api.forward(qd, kd, vd, w.grid, w.tile, topk, **gu.geo(w))
    assert torch.equal(idx, idx2) and torch.equal(o, o2) and torch.equal(lse, lse2)
    gu.check_selection(idx.cpu().numpy(), gu.oracle_scores(q, k, w), topk)


# Score kernel per head size: up to 128 key tiles the narrow kernel with
# 128-key passes (the small cases and Wan-5B), 129..256 with 256-key passes,
# 257..768 the wide kernel with a 3-deep ring, 769..1024 with a 2-deep one,
# larger ones the narrow kernel again, up to the 1536-tile limit; ragged on
# every axis.
MANY_TILES = [
    Workload("tiles150", 1, 2, (10, 19, 40), 64, (4, 4, 4), 20, "field"),
    Workload("tiles768", 1, 1, (15, 47, 63), 64, (4, 4, 4), 48, "field"),
    Workload("tiles960", 1, 2, (19, 45, 62), 64, (4, 4, 4), 60, "field"),
    Workload("tiles1024", 1, 1, (15, 61, 62), 128, (4, 4, 4), 64, "field"),
    Workload("tiles1536", 1, 1, (23, 61, 62), 64, (4, 4, 4), 96),
]


@pytest.mark.parametrize("w", MANY_TILES, ids=lambda w: w.name)
def test_many_tiles(w):
    assert vo.num_tiles(w.grid, w.tile) == int(w.name[5:])
    rep = _full_case(w)
    print(w.name, rep)


@pytest.mark.parametrize("kind", ["normal", "field"])
def test_full_size_sweep(kind):
    base = [s for s in SWEEP if s.kind == kind][0]
    rep = _full_case(base, topks=[s.topk for s in SWEEP if s.kind == kind])
    print("sweep", kind, rep)


def test_full_size_sweep_all_tiles_is_dense():
    """Wan-5B shape, topk 120 = every tile: sampled rows equal dense attention."""
    w = WAN5B.with_(topk=120)
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=1)
    idx = api.select(qd, kd, w.grid, w.tile, 120)
    o, lse = api.attn_fwd(qd, kd, vd, idx, w.grid, w.tile)
    gu.assert_no_device_error()
    rng = np.random.default_rng(0)
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    scale = w.d ** -0.5
    for bh in (0, 17):
        rows = np.concatenate([[0, w.N - 1], rng.choice(w.N, 30, replace=False)])
        Q, K, V = (vo.widen(x[0, bh], w.dtype) for x in (q, k, v))
        Od, Ld = vo.dense_bruteforce(Q[rows], K, V, scale)
        e = np.abs(og[0, bh][rows] - Od)
        assert e.max() <= gu.O_MAX_ABS and e.mean() <= gu.O_MEAN_ABS
        assert np.abs(lg[0, bh][rows] - Ld).max() <= gu.LSE_ABS


HOST_CASES = [
    (Workload("host_pipe", 2, 3, (9, 20, 20), 128, (4, 8, 8), 5), 1),
    (Workload("host_pipe", 2, 3, (9, 20, 20), 128, (4, 8, 8), 5), 2),
    (Workload("host_pipe", 2, 3, (9, 20, 20), 128, (4, 8, 8), 5), 5),
    # [B, N, H, d]: chunks are strided blocks of one batch's heads (3 heads in chunks of 2: a short last one)
    (Workload("host_bnhd", 2, 3, (6, 10, 14), 128, (4, 4, 4), 5, "field", layout="bnhd"), 2),
    # own key/value grid and tile, always-kept prefix tiles, fp16, [B, N, H, d]
    (Workload("host_kv_prefix", 2, 2, (8, 12, 16), 64, (4, 4, 4), 12, "field", grid_k=(12, 12, 16),
              prefix_tiles=12, layout="bnhd", dtype="f16"), 1),
]


@pytest.mark.parametrize("w,chunk", HOST_CASES, ids=[f"{w.name}-c{c}" for w, c in HOST_CASES])
def test_forward_host_matches_device_path(w, chunk):
    """vsa_forward_host (host buffers in and out) gives the device path's bits,
    and those match the oracle."""
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=6)
    kw = dict(grid_k=w.grid_k, tile_k=w.tile_k, layout=w.layout, prefix_tiles=w.prefix_tiles)
    o_ref, l_ref, i_ref = api.forward(qd, kd, vd, w.grid, w.tile, w.topk, **kw)
    hq, hk, hv = (qd.cpu().pin_memory(), kd.cpu().pin_memory(), vd.cpu().pin_memory())
    o, l, i = api.forward_host(hq, hk, hv, w.grid, w.tile, w.topk, chunk_heads=chunk, **kw)
    gu.assert_no_device_error()
    assert torch.equal(i, i_ref.cpu())
    assert torch.equal(o.view(torch.int16), o_ref.cpu().view(torch.int16))
    assert torch.equal(l, l_ref.cpu())
    gu.check_selection(i.numpy(), gu.oracle_scores(q, k, w), w.topk)
    gu.check_attention(o, l, q, k, v, w, i.numpy(), w.d ** -0.5)
