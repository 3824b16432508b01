"""Pins for the CPU oracle: values and properties fixed by the pages and by
mathematics, not by the oracle itself.  No GPU needed.

Sources: FastVideo VSA user guide (routing log in "Wan top-k behavior"; block
sizes in "Verify routing and fallback"); fastbsa 0.1.0 page ("How it works":
validation against dense attention).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import loops
from oracle import vsa_oracle as vo
from block_sparse_video_tile_b200 import synth
from block_sparse_video_tile_b200.workloads import ALL, LONGCAT, TINY, WAN14B, WAN5B

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(shape, seed):
    """float64 values that are exactly representable in bfloat16."""
    rng = np.random.default_rng(seed)
    return vo.bf16_to_f64(synth.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32)))


# ------------------------------------------------------------------ geometry
def test_routing_log_example():
    g = _golden("wan_routing_log.json")
    grid, blk = tuple(g["dit_seq_shape"]), tuple(g["block_size"])
    assert math.prod(grid) == g["seq_len"]
    assert vo.num_tiles(grid, blk) == g["num_blocks"]
    # floor tiling would drop the partial edge blocks: 7 * 2 * 5 = 70 != 120
    assert math.prod(x // b for x, b in zip(grid, blk)) != g["num_blocks"]
    assert round(100.0 * g["topk"] / g["num_blocks"], 1) == g["keep_ratio_percent"]


def test_block_sizes():
    g = _golden("block_sizes.json")
    assert math.prod(g["wan_block"]) == g["wan_block_tokens"]
    assert math.prod(g["h3_block"]) == g["h3_block_tokens"]
    # the LongCat-like workload keeps (1 - sparsity) of its 720 blocks
    nT = vo.num_tiles(LONGCAT.grid, LONGCAT.tile)
    assert nT == 720 and nT * (1 - g["fastbsa_sparsity"]) == LONGCAT.topk


@pytest.mark.parametrize("w,expect", [
    (TINY, {64: 8}),
    (WAN5B, {256: 70, 192: 45, 144: 5}),
    (WAN14B, {256: 240, 128: 60}),
    (LONGCAT, {64: 720}),
])
def test_block_token_counts(w, expect):
    toks = vo.tile_tokens(w.grid, w.tile)
    counts = {}
    for t in toks:
        counts[len(t)] = counts.get(len(t), 0) + 1
    assert counts == expect
    # the blocks partition the token range exactly
    allt = np.concatenate(toks)
    assert allt.size == w.N and np.array_equal(np.sort(allt), np.arange(w.N))


def test_block_raster_order():
    grid, tile = (5, 6, 7), (2, 4, 4)
    toks = vo.tile_tokens(grid, tile)
    nt, nh, nw = vo.tiles_per_axis(grid, tile)
    assert (nt, nh, nw) == (3, 2, 2)
    for j, t in enumerate(toks):
        bt, bh, bw = j // (nh * nw), (j // nw) % nh, j % nw
        n = t[0]                                  # first token = block origin
        assert (n // (6 * 7), (n // 7) % 6, n % 7) == (bt * 2, bh * 4, bw * 4)


# ------------------------------------------------------------------- pooling
def test_pool_constant_per_block_partial_edges():
    grid, tile = (5, 6, 7), (4, 4, 4)               # partial on every axis
    toks = vo.tile_tokens(grid, tile)
    N, d = math.prod(grid), 3
    consts = np.arange(len(toks) * d, dtype=np.float64).reshape(len(toks), d) - 5.0
    X = np.empty((N, d))
    for j, t in enumerate(toks):
        X[t] = consts[j]
    np.testing.assert_array_equal(vo.pool(X, grid, tile), consts)


def test_pool_weighted_sum_invariant():
    grid, tile = (5, 6, 7), (4, 4, 4)
    X = _rand((math.prod(grid), 5), 1)
    counts = np.array([len(t) for t in vo.tile_tokens(grid, tile)], dtype=np.float64)
    np.testing.assert_allclose((counts[:, None] * vo.pool(X, grid, tile)).sum(0), X.sum(0),
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------- scores and top-k
def _hand_example():
    # grid (1, 1, 6), blocks (1, 1, 2): three blocks along x, d = 2
    grid, tile = (1, 1, 6), (1, 1, 2)
    qbar = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    kbar = np.array([[2.0, 0.0], [0.0, 3.0], [-1.0, 1.0]])
    Q = np.repeat(qbar, 2, axis=0)
    K = np.repeat(kbar, 2, axis=0)
    return grid, tile, Q, K


def test_scores_hand_example():
    grid, tile, Q, K = _hand_example()
    idx, s, near = vo.select_head(Q, K, grid, tile, 2)
    np.testing.assert_array_equal(s, [[2, 0, -1], [0, 3, 1], [2, 3, 0]])
    np.testing.assert_array_equal(idx, [[0, 1], [1, 2], [0, 1]])
    assert not near.any()


def test_ties_go_to_lower_index():
    grid, tile = (1, 1, 8), (1, 1, 2)             # 4 blocks
    Q = np.ones((8, 2))
    K = np.repeat(np.array([[1.0, 0.0], [0.5, 0.5], [0.5, 0.5], [0.0, 0.0]]), 2, axis=0)
    # scores per row: [1, 1, 1, 0] -> blocks 0, 1, 2 tie; topk 2 keeps 0 and 1
    idx, _, near = vo.select_head(Q, K, grid, tile, 2)
    assert (idx == [0, 1]).all()
    assert near.all()
    idx3, _, _ = vo.select_head(Q, K, grid, tile, 3)
    assert (idx3 == [0, 1, 2]).all()


def test_all_blocks_kept():
    grid, tile = (5, 6, 7), (4, 4, 4)
    Q, K = _rand((210, 4), 2), _rand((210, 4), 3)
    nT = vo.num_tiles(grid, tile)
    idx, _, near = vo.select_head(Q, K, grid, tile, nT)
    assert (idx == np.arange(nT)).all() and not near.any()


def test_topk_range_rejected():
    grid, tile = (4, 4, 4), (2, 2, 2)
    Q = K = np.ones((64, 2))
    for bad in (0, -1, 9):
        with pytest.raises(ValueError):
            vo.select_head(Q, K, grid, tile, bad)


def test_positive_scale_leaves_selection():
    grid, tile = (5, 6, 7), (2, 2, 4)
    Q, K = _rand((210, 8), 4), _rand((210, 8), 5)
    a, _, _ = vo.select_head(Q, K, grid, tile, 5)
    b, _, _ = vo.select_head(3.7 * Q, K, grid, tile, 5)
    assert (a == b).all()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_vs_rank_bruteforce(seed):
    """Rank counting in plain Python vs the sort in NumPy, with forced ties."""
    grid, tile = (4, 4, 6), (2, 2, 2)
    Q, K = _rand((96, 3), 10 + seed), _rand((96, 3), 20 + seed)
    toks = vo.tile_tokens(grid, tile)
    K[toks[5]] = K[toks[2]]                       # blocks 2 and 5 score identically
    for topk in (1, 3, 6, 12):
        idx, _, _ = vo.select_head(Q, K, grid, tile, topk)
        lidx, _ = loops.select(Q.tolist(), K.tolist(), grid, tile, topk)
        assert idx.tolist() == lidx


def test_near_tie_band_and_validity():
    s = np.array([5.0, 1.0 + 1e-9, 1.0, -2.0])
    rel, delta = vo.tie_gap(s, 2)
    assert rel < vo.NEAR_TIE_REL and delta > 1e-9
    assert vo.selection_is_valid(np.array([0, 1]), s, 2)
    assert vo.selection_is_valid(np.array([0, 2]), s, 2)      # the other side of the tie
    assert not vo.selection_is_valid(np.array([0, 3]), s, 2)  # outside the band
    assert not vo.selection_is_valid(np.array([1, 2]), s, 2)
    assert not vo.selection_is_valid(np.array([2, 0]), s, 2)  # not ascending
    s2 = np.array([5.0, 2.0, 1.0, -2.0])
    assert vo.tie_gap(s2, 2)[0] >= vo.NEAR_TIE_REL
    assert not vo.selection_is_valid(np.array([0, 2]), s2, 2)


# ----------------------------------------------------------------- attention
def _head(grid, d, seed):
    N = math.prod(grid)
    return _rand((N, d), seed), _rand((N, d), seed + 1), _rand((N, d), seed + 2)


@pytest.mark.parametrize("grid,tile", [((8, 8, 8), (4, 4, 4)), ((5, 6, 7), (4, 4, 4)),
                                       ((3, 5, 9), (2, 4, 8))])
def test_all_blocks_equals_dense(grid, tile):
    Q, K, V = _head(grid, 16, 30)
    nT = vo.num_tiles(grid, tile)
    idx = np.tile(np.arange(nT), (nT, 1))
    scale = 16 ** -0.5
    O, L = vo.attend_head(Q, K, V, grid, tile, idx, scale)
    Od, Ld = vo.dense_bruteforce(Q, K, V, scale)
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-12)


def test_dense_vs_library_sdpa():
    Q, K, V = _head((4, 4, 8), 32, 40)
    scale = 32 ** -0.5
    Od, Ld = vo.dense_bruteforce(Q, K, V, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        scale=scale)[0].numpy()
    np.testing.assert_allclose(Od, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Ld, logsumexp(scale * Q @ K.T, axis=1), rtol=0, atol=1e-12)


def test_zero_scale_is_mean_of_kept_values():
    grid, tile = (5, 6, 7), (4, 4, 4)
    Q, K, V = _head(grid, 8, 50)
    toks = vo.tile_tokens(grid, tile)
    nT = len(toks)
    rng = np.random.default_rng(0)
    idx = np.sort(np.stack([rng.choice(nT, 3, replace=False) for _ in range(nT)]), axis=1)
    O, L = vo.attend_head(Q, K, V, grid, tile, idx, 0.0)
    for i in range(nT):
        keys = np.concatenate([toks[j] for j in idx[i]])
        np.testing.assert_allclose(O[toks[i]], np.broadcast_to(V[keys].mean(0), O[toks[i]].shape),
                                   rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[toks[i]], math.log(keys.size), rtol=0, atol=1e-12)


def test_constant_values_pass_through():
    grid, tile = (5, 6, 7), (4, 4, 4)
    Q, K, _ = _head(grid, 8, 60)
    c = np.linspace(-2, 3, 8)
    V = np.tile(c, (Q.shape[0], 1))
    nT = vo.num_tiles(grid, tile)
    idx = np.tile(np.arange(2), (nT, 1))
    O, _ = vo.attend_head(Q, K, V, grid, tile, idx, 0.7)
    np.testing.assert_allclose(O, np.tile(c, (Q.shape[0], 1)), rtol=0, atol=1e-12)


def test_lse_normalises_weights():
    grid, tile = (5, 6, 7), (4, 4, 4)
    Q, K, V = _head(grid, 8, 70)
    toks = vo.tile_tokens(grid, tile)
    nT = len(toks)
    idx = np.tile(np.array([0, 3, 5]), (nT, 1))
    scale = 0.9
    _, L = vo.attend_head(Q, K, V, grid, tile, idx, scale)
    keys = np.concatenate([toks[j] for j in (0, 3, 5)])
    for n in range(Q.shape[0]):
        z = [scale * float(np.dot(Q[n], K[m])) for m in keys]
        assert abs(sum(math.exp(v - L[n]) for v in z) - 1.0) < 1e-12


def test_permutation_inside_blocks():
    grid, tile = (4, 4, 8), (2, 2, 4)
    Q, K, V = _head(grid, 8, 80)
    toks = vo.tile_tokens(grid, tile)
    rng = np.random.default_rng(3)
    perm = np.arange(Q.shape[0])
    for t in toks:                                 # shuffle tokens within each block
        perm[t] = t[rng.permutation(t.size)]
    idx, s, _ = vo.select_head(Q, K, grid, tile, 3)
    idx2, s2, _ = vo.select_head(Q[perm], K[perm], grid, tile, 3)
    np.testing.assert_allclose(s, s2, rtol=0, atol=1e-12)
    assert (idx == idx2).all()
    O, L = vo.attend_head(Q, K, V, grid, tile, idx, 0.5)
    O2, L2 = vo.attend_head(Q[perm], K[perm], V[perm], grid, tile, idx, 0.5)
    np.testing.assert_allclose(O2, O[perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L[perm], rtol=0, atol=1e-12)


def test_loops_agree_on_tiny():
    """The NumPy oracle against the pure-Python restatement on the Tiny workload."""
    q, k, v = synth.make_qkv(TINY.B, TINY.H, TINY.grid, TINY.d, seed=0)
    scale = TINY.d ** -0.5
    for h in range(TINY.H):
        Q, K, V = (vo.bf16_to_f64(x[0, h]) for x in (q, k, v))
        idx, s, _ = vo.select_head(Q, K, TINY.grid, TINY.tile, TINY.topk)
        lidx, ls = loops.select(Q.tolist(), K.tolist(), TINY.grid, TINY.tile, TINY.topk)
        assert idx.tolist() == lidx
        np.testing.assert_allclose(s, np.array(ls), rtol=1e-12, atol=1e-15)
        O, L = vo.attend_head(Q, K, V, TINY.grid, TINY.tile, idx, scale)
        lO, lL = loops.attend(Q.tolist(), K.tolist(), V.tolist(), TINY.grid, TINY.tile, lidx, scale)
        np.testing.assert_allclose(O, np.array([lO[n] for n in range(TINY.N)]), rtol=0, atol=1e-12)
        np.testing.assert_allclose(L, np.array([lL[n] for n in range(TINY.N)]), rtol=0, atol=1e-12)


def test_workload_table():
    """Block counts and keep ratios of every workload (closed form)."""
    expect = {"tiny": 8, "wan5b": 120, "wan14b": 300, "longcat": 720}
    for name, nT in expect.items():
        w = ALL[name]
        assert vo.num_tiles(w.grid, w.tile) == nT
        assert 0 < w.topk <= nT
    for w in ALL.values():
        if w.name.startswith("sweep"):
            assert vo.num_tiles(w.grid, w.tile) == 120 and w.topk in (8, 16, 32, 64, 120)


def test_bf16_widening_textbook_values():
    """bfloat16 encodings (the upper half of a float32): 1.0, -2.0, the largest
    finite 0x7F7F = (2 - 2^-7) * 2^127, the smallest subnormal 2^-133, 1/3
    rounded; and round-to-nearest-even when narrowing float32 to bfloat16."""
    bits = np.array([0x3F80, 0xC000, 0x7F7F, 0x0001, 0x3EAB], dtype=np.uint16)
    w = vo.bf16_to_f64(bits)
    np.testing.assert_array_equal(w[:4], [1.0, -2.0, (2 - 2.0 ** -7) * 2.0 ** 127, 2.0 ** -133])
    assert abs(w[4] - 1 / 3) < 2 ** -9
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties round to the even one (1.0)
    assert synth.f32_to_bf16_bits(np.array([1 + 2 ** -8], np.float32))[0] == 0x3F80
    assert synth.f32_to_bf16_bits(np.array([1 + 3 * 2 ** -8], np.float32))[0] == 0x3F82
    assert synth.f32_to_bf16_bits(np.array([-1.5], np.float32))[0] == 0xBFC0


def test_f16_widening_textbook_values():
    """IEEE binary16 encodings: 1.0, -2.0, the largest finite 65504, the
    smallest subnormal 2^-24, and round-to-nearest-even at a tie."""
    bits = np.array([0x3C00, 0xC000, 0x7BFF, 0x0001, 0x3555], dtype=np.uint16)
    np.testing.assert_array_equal(vo.f16_to_f64(bits)[:4], [1.0, -2.0, 65504.0, 2.0 ** -24])
    assert abs(vo.f16_to_f64(bits)[4] - 1 / 3) < 2 ** -11
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: ties round to the even one (1.0)
    assert synth.f32_to_f16_bits(np.array([1 + 2 ** -11], np.float32))[0] == 0x3C00
    assert synth.f32_to_f16_bits(np.array([1 + 3 * 2 ** -11], np.float32))[0] == 0x3C02


# ------------------------------------- separate key/value grid, sparsity (fastbsa page, "Use")
KV_CASES = [
    # (query grid, query tile, key/value grid, key/value tile); partial edge tiles on both sides
    ((3, 5, 6), (2, 2, 2), (5, 4, 7), (2, 2, 2)),
    ((4, 4, 4), (2, 2, 2), (6, 3, 5), (4, 2, 1)),
]


@pytest.mark.parametrize("grid_q,tile_q,grid_k,tile_k", KV_CASES)
def test_kv_grid_all_blocks_equals_dense(grid_q, tile_q, grid_k, tile_k):
    # keeping every key/value block is dense attention of the Nq queries over
    # all Nk keys, whatever the two tilings (closed form, no tiles in the reference)
    Nq, Nk, d = math.prod(grid_q), math.prod(grid_k), 8
    Q, K, V = _rand((Nq, d), 21), _rand((Nk, d), 22), _rand((Nk, d), 23)
    nTq, nTk = vo.num_tiles(grid_q, tile_q), vo.num_tiles(grid_k, tile_k)
    idx, s, _ = vo.select_head(Q, K, grid_q, tile_q, nTk, grid_k, tile_k)
    assert s.shape == (nTq, nTk)
    assert (idx == np.arange(nTk)).all()
    O, L = vo.attend_head(Q, K, V, grid_q, tile_q, idx, 0.3, grid_k=grid_k, tile_k=tile_k)
    Od, Ld = vo.dense_bruteforce(Q, K, V, 0.3)
    np.testing.assert_allclose(O, Od, atol=1e-12)
    np.testing.assert_allclose(L, Ld, atol=1e-12)


def test_kv_pool_uses_kv_tiles():
    # K constant on each of its own (partial-edged) tiles: its means are those constants
    grid_q, tile_q, grid_k, tile_k = KV_CASES[1]
    d = 6
    rng = np.random.default_rng(5)
    toks = vo.tile_tokens(grid_k, tile_k)
    vals = rng.standard_normal((len(toks), d))
    K = np.zeros((math.prod(grid_k), d))
    for j, t in enumerate(toks):
        K[t] = vals[j]
    Q = _rand((math.prod(grid_q), d), 24)
    _, s, _ = vo.select_head(Q, K, grid_q, tile_q, 1, grid_k, tile_k)
    assert s.shape == (vo.num_tiles(grid_q, tile_q), len(toks))
    np.testing.assert_allclose(s, vo.pool(Q, grid_q, tile_q) @ vals.T, atol=1e-12)


def test_topk_from_sparsity():
    # fastbsa page, "Use": sparsity=0.9375 keeps one block in 16
    assert vo.topk_from_sparsity(720, 0.9375) == 45
    assert vo.topk_from_sparsity(16, 0.9375) == 1
    # exact keep fractions need no rounding
    for n, k in ((120, 64), (300, 30), (720, 45), (8, 2), (1536, 1536)):
        assert vo.topk_from_sparsity(n, 1.0 - k / n) == k
    for n in (1, 7, 120):
        assert vo.topk_from_sparsity(n, 0.0) == n
    # reading: halves round up, and at least one block is kept
    assert vo.topk_from_sparsity(10, 0.85) == 2
    assert vo.topk_from_sparsity(10, 0.99) == 1
    for bad in (1.0, -0.1, 1.5):
        with pytest.raises(ValueError):
            vo.topk_from_sparsity(10, bad)


# ----------------------------- always-kept prefix blocks (user guide, "Choose top-k": H3)
def _ranked(scores, k):
    """The k best of (index, score) pairs, ties to the lower index, by a plain sort."""
    return [j for _, j in sorted((-sc, j) for j, sc in scores)[:k]]


@pytest.mark.parametrize("prefix,topk", [(0, 5), (3, 5), (3, 3), (6, 9)])
def test_prefix_blocks_always_kept(prefix, topk):
    # prefix blocks get the lowest means on purpose: plain top-k would drop them
    grid, tile, d = (4, 6, 6), (2, 2, 2), 5                  # 2 x 3 x 3 = 18 blocks
    rng = np.random.default_rng(9)
    Q = _rand((math.prod(grid), d), 31)
    K = _rand((math.prod(grid), d), 32)
    toks = vo.tile_tokens(grid, tile)
    qm = vo.pool(Q, grid, tile).mean(axis=0)
    for j in range(prefix):
        K[toks[j]] = -10.0 * qm / max(np.linalg.norm(qm), 1e-9) + 0.01 * rng.standard_normal((len(toks[j]), d))
    idx, s, near = vo.select_head(Q, K, grid, tile, topk, prefix=prefix)
    raw = vo.tile_scores(vo.pool(Q, grid, tile), vo.pool(K, grid, tile))
    for i in range(len(toks)):
        rest = _ranked([(j, raw[i, j]) for j in range(prefix, len(toks))], topk - prefix)
        assert idx[i].tolist() == sorted(list(range(prefix)) + rest)
    if prefix:
        # the inputs are such that plain top-k would leave prefix blocks out
        plain, _, _ = vo.select_head(Q, K, grid, tile, topk)
        assert any(not set(range(prefix)) <= set(plain[i].tolist()) for i in range(len(toks)))
    # the tie band only looks at the blocks that compete
    for i in range(len(toks)):
        rel, _ = vo.tie_gap(s[i], topk)
        if topk == prefix:
            assert rel == math.inf
        else:
            ref, _ = vo.tie_gap(raw[i, prefix:], topk - prefix)
            assert rel == pytest.approx(ref, rel=1e-12, abs=1e-300) or (math.isinf(rel) and math.isinf(ref))


def test_prefix_range_rejected():
    grid, tile = (4, 4, 4), (2, 2, 2)
    Q = _rand((64, 4), 33)
    with pytest.raises(ValueError):
        vo.select_head(Q, Q, grid, tile, 2, prefix=3)       # topk < prefix
    with pytest.raises(ValueError):
        vo.select_head(Q, Q, grid, tile, 8, prefix=9)       # prefix > nT
    assert vo.topk_from_sparsity(8, 0.99, prefix=3) == 3


# ------------------------------------------------------------ coarse branch
# The pooled coarse branch (FastVideo VSA user guide, "Checkpoint behavior":
# a learned gate_compress compensation added to the sparse branch) has no
# formula on the pages; the oracle's reading is tile-level attention over the
# blocks' mean rows, added through a caller-given gate.  These pins fix that
# reading by closed forms and by the pure-Python restatement.
RAGGED_COARSE = ((5, 6, 7), (2, 4, 4))      # 3 x 2 x 2 blocks, partial on every axis


def _block_means_loops(X, grid, tile):
    """Mean rows of every block, from the pure-Python block lists."""
    return np.array([loops.mean_rows(X.tolist(), grid, toks) for toks in loops.blocks(grid, tile)])


@pytest.mark.parametrize("grid, tile", [(TINY.grid, TINY.tile), RAGGED_COARSE])
def test_coarse_uniform_keys_average_block_values(grid, tile):
    """All key blocks with the same mean (or a zero scale): every block gets
    the same weight, so o_coarse is the plain average of the blocks' mean V
    rows -- each partial block counting once, not by its token count."""
    N = math.prod(grid)
    Q, V = _rand((N, 8), 1), _rand((N, 8), 2)
    K = np.tile(_rand((1, 8), 3), (N, 1))
    expect = _block_means_loops(V, grid, tile).mean(axis=0)
    oc = vo.coarse_head(Q, K, V, grid, tile, 0.7)
    np.testing.assert_allclose(oc, np.broadcast_to(expect, oc.shape), rtol=0, atol=1e-12)
    oc0 = vo.coarse_head(Q, _rand((N, 8), 4), V, grid, tile, 0.0)
    np.testing.assert_allclose(oc0, np.broadcast_to(expect, oc0.shape), rtol=0, atol=1e-12)
    if N % math.prod(tile):
        # partial blocks: a zero-padded mean over the full block volume would differ
        assert not np.allclose(expect, V.sum(axis=0) / (len(loops.blocks(grid, tile)) * math.prod(tile)))


def test_coarse_dominant_block_selects_its_values():
    """One key block whose mean points along every query mean, with a large
    scale: its weight is 1 - O(nT e^-60), so o_coarse is that block's mean V."""
    grid, tile = RAGGED_COARSE
    N = math.prod(grid)
    Q = np.zeros((N, 8))
    Q[:, 0] = 1.0
    K = np.zeros((N, 8))
    star = 5
    toks = loops.blocks(grid, tile)[star]
    for t, y, x in toks:
        K[(t * grid[1] + y) * grid[2] + x, 0] = 60.0
    V = _rand((N, 8), 5)
    oc = vo.coarse_head(Q, K, V, grid, tile, 1.0)
    expect = _block_means_loops(V, grid, tile)[star]
    np.testing.assert_allclose(oc, np.broadcast_to(expect, oc.shape), rtol=0, atol=1e-12)


def test_coarse_constant_values_pass_through():
    """V equal to one row c everywhere: the softmax weights sum to 1, so
    o_coarse = c for every query block."""
    grid, tile = RAGGED_COARSE
    N = math.prod(grid)
    c = _rand((1, 8), 6)
    oc = vo.coarse_head(_rand((N, 8), 7), _rand((N, 8), 8), np.tile(c, (N, 1)), grid, tile, 0.9)
    np.testing.assert_allclose(oc, np.broadcast_to(c, oc.shape), rtol=0, atol=1e-12)


def test_coarse_scale_matters():
    """The scale multiplies the tile scores before the softmax: a larger
    scale sharpens the weights (an unscaled oracle would give equal outputs)."""
    grid, tile = RAGGED_COARSE
    N = math.prod(grid)
    Q, K, V = _rand((N, 8), 9), _rand((N, 8), 10), _rand((N, 8), 11)
    a = vo.coarse_head(Q, K, V, grid, tile, 0.1)
    b = vo.coarse_head(Q, K, V, grid, tile, 10.0)
    assert np.abs(a - b).max() > 1e-3


@pytest.mark.parametrize("grid, tile", [(TINY.grid, TINY.tile), RAGGED_COARSE])
def test_coarse_and_gate_vs_loops(grid, tile):
    """NumPy coarse branch and gated output against the pure-Python
    restatement (its own block lists, dot products and exp)."""
    N = math.prod(grid)
    d = 8
    Q, K, V, G, O = (_rand((N, d), s) for s in (12, 13, 14, 15, 16))
    oc = vo.coarse_head(Q, K, V, grid, tile, 0.35)
    loc = loops.coarse(Q.tolist(), K.tolist(), V.tolist(), grid, tile, 0.35)
    np.testing.assert_allclose(oc, np.array(loc), rtol=0, atol=1e-12)
    out = vo.gated_output(O, G, oc, grid, tile)
    lout = loops.gated(O.tolist(), G.tolist(), loc, grid, tile)
    np.testing.assert_allclose(out, np.array([lout[n] for n in range(N)]), rtol=0, atol=1e-12)


def test_gate_zero_is_identity_and_gate_is_linear():
    grid, tile = RAGGED_COARSE
    N = math.prod(grid)
    O, G = _rand((N, 8), 17), _rand((N, 8), 18)
    oc = _rand((len(loops.blocks(grid, tile)), 8), 19)
    assert np.array_equal(vo.gated_output(O, np.zeros_like(G), oc, grid, tile), O)
    one = vo.gated_output(O, G, oc, grid, tile) - O
    two = vo.gated_output(O, 2 * G, oc, grid, tile) - O
    np.testing.assert_allclose(two, 2 * one, rtol=0, atol=1e-12)
