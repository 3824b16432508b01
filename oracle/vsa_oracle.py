"""Plain float64 CPU oracle for VSA-style 3-D block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only the tests, the package's smoke check and the benchmark's CPU-baseline leg
call it.  It shares no code with the CUDA library (its own geometry, its own
pooling, scoring, selection and softmax), and takes its inputs as bfloat16 or
float16 bit patterns widened exactly to float64.

What it computes, and where the pages fix each step:

1. Tiling (FastVideo VSA user guide, intro and "Wan top-k behavior"): the
   post-patch latent grid (T, Hh, W) is cut into spatio-temporal blocks of
   (tt, th, tw) tokens; the number of blocks per axis is the ceiling of
   extent / block, so edge blocks are partial -- the guide's routing log gives
   (31, 22, 40) with (4, 8, 8) blocks -> num_blocks = 120 = 8 * 3 * 5.
   Blocks are numbered in raster order over block coordinates (t-major, then
   y, then x), the same order as tokens.
2. Scoring (guide intro: "for every query block, VSA scores the key/value
   blocks"): each block is summarised by the mean of its Q rows (resp. K rows)
   over its valid tokens; the score of (query block i, key block j) is the dot
   product of the two means.  Reading: mean over valid tokens only (a partial
   block divides by its own token count), and no scale factor (a positive
   scale changes neither the order nor the relative gaps).
3. Selection (guide "Wan top-k behavior": top-k counts key/value blocks per
   query block, 0 < topk <= num_blocks): keep the topk largest scores; equal
   scores are broken by the lower block index; the kept list is stored in
   ascending block order.
4. Attention (guide intro and "Verify routing and fallback": non-causal
   self-attention, no mask, scale head_size ** -0.5 by default): for every
   token of query block i, exact softmax attention over the tokens of the kept
   blocks; LSE is the natural log of the softmax denominator.
5. Dense reference (fastbsa page, "How it works": outputs are validated
   against dense attention): plain softmax attention over all N tokens, with no
   tiles at all.  With topk == num_blocks (all blocks kept) step 4 equals it.
6. Separate key/value grid (fastbsa page, "Use": latent_shape_q /
   latent_shape_k and chunk_3d_shape_q / chunk_3d_shape_k): the query tokens
   are tiled with the query grid and chunk, the key/value tokens with their
   own; steps 2-4 then run with query tiles on one side and key/value tiles on
   the other (scores nTq x nTk, top-k over nTk).
7. Sparsity (fastbsa page, "Use": sparsity=0.9375): the fraction of key/value
   blocks left out.  Reading: topk = round((1 - sparsity) * nTk), halves
   rounding up, clamped to [max(1, P), nTk] (0.9375 of 720 blocks keeps 45).
8. Always-kept prefix blocks (user guide, "Choose top-k": H3 "keeps all prefix
   blocks").  Reading: the first P key/value blocks in raster order are in
   every query block's kept list whatever their scores (their scores count
   as +inf for the selection) and count toward topk; the other topk - P are
   the best-scoring of the rest.
9. Pooled coarse branch (user guide, "Checkpoint behavior": checkpoints
   that carry learned `to_gate_compress` weights add a gated compensation to
   the sparse branch; without them the sparse branch runs alone).  The pages
   name the branch but not its math -- parity unpinned by the pages.
   Reading: attention at tile granularity.  Each query block's mean row
   attends over every key/value block's mean row with the fine branch's
   scale, softmax over all key/value blocks (each block one entry, whatever
   its token count), values = the blocks' mean V rows; the result
   o_coarse[i] is added to every token n of query block i through a gate
   the caller supplies (the projection's output, same shape as O):
   O[n] = O_sparse[n] + gate[n] * o_coarse[i].
"""
from __future__ import annotations

import math

import numpy as np

NEAR_TIE_REL = 1e-4      # relative k-th / (k+1)-th score gap that counts as a near-tie
EPS_ROW_REL = 1e-6       # guards the relative gap when both scores are ~0


# ---------------------------------------------------------------- conversions
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) exactly to float64."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen IEEE half-precision bit patterns (uint16) exactly to float64."""
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def widen(bits: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    """Exact float64 values of 16-bit inputs ("bf16" or "f16" bit patterns)."""
    return f16_to_f64(bits) if dtype == "f16" else bf16_to_f64(bits)


# ------------------------------------------------------------------- geometry
def tiles_per_axis(grid, tile):
    """Blocks per axis: ceil(extent / block extent)."""
    return tuple(-(-g // t) for g, t in zip(grid, tile))


def num_tiles(grid, tile) -> int:
    nt, nh, nw = tiles_per_axis(grid, tile)
    return nt * nh * nw


def tile_tokens(grid, tile):
    """Raster token indices of every block, in block raster order.

    Returns a list of 1-D int64 arrays; list entry j holds the tokens
    n = (t * Hh + y) * W + x of block j, in raster order inside the block.
    """
    T, Hh, W = grid
    tt, th, tw = tile
    nt, nh, nw = tiles_per_axis(grid, tile)
    out = []
    for bt in range(nt):
        ts = np.arange(bt * tt, min(T, (bt + 1) * tt))
        for bh in range(nh):
            ys = np.arange(bh * th, min(Hh, (bh + 1) * th))
            for bw in range(nw):
                xs = np.arange(bw * tw, min(W, (bw + 1) * tw))
                n = (ts[:, None, None] * Hh + ys[None, :, None]) * W + xs[None, None, :]
                out.append(n.reshape(-1).astype(np.int64))
    return out


# -------------------------------------------------------------------- scoring
def pool(X: np.ndarray, grid, tile) -> np.ndarray:
    """Per-block mean of the rows of X ([N, d] float64) over valid tokens."""
    return np.stack([X[tok].mean(axis=0) for tok in tile_tokens(grid, tile)])


def tile_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """s[i, j] = qbar_i . kbar_j (float64)."""
    return qbar @ kbar.T


def topk_row(s_row: np.ndarray, topk: int) -> np.ndarray:
    """The topk largest entries of one score row, ties -> lower index, ascending."""
    order = np.lexsort((np.arange(s_row.shape[0]), -s_row))   # by (-s, j)
    return np.sort(order[:topk])


def tie_gap(s_row: np.ndarray, topk: int):
    """(relative gap, absolute band delta) between the k-th and (k+1)-th scores.

    Returns (inf, 0) when topk == number of blocks (nothing is left out) or
    when the cut falls next to an always-kept (+inf) block.
    """
    nT = s_row.shape[0]
    if topk >= nT:
        return math.inf, 0.0
    srt = np.sort(s_row)[::-1]
    a, b = srt[topk - 1], srt[topk]
    if not (np.isfinite(a) and np.isfinite(b)):
        return math.inf, 0.0
    finite = np.abs(s_row[np.isfinite(s_row)])
    denom = max(abs(a), abs(b), EPS_ROW_REL * float(finite.max()))
    if denom == 0.0:
        return 0.0, 0.0
    return abs(a - b) / denom, NEAR_TIE_REL * denom


def keep_prefix(scores: np.ndarray, prefix: int) -> np.ndarray:
    """Scores as the selection sees them: the first ``prefix`` key/value blocks at +inf."""
    s = np.array(scores, dtype=np.float64, copy=True)
    s[..., :prefix] = math.inf
    return s


def select_head(Q: np.ndarray, K: np.ndarray, grid, tile, topk: int, grid_k=None, tile_k=None, prefix: int = 0):
    """One head: (idx [nTq, topk] int32 ascending, scores [nTq, nTk], near_tie [nTq] bool).

    K is tiled with grid_k / tile_k (default: the query grid / tile).  The
    scores returned are the selection's: the first ``prefix`` blocks at +inf.
    """
    grid_k = grid if grid_k is None else grid_k
    tile_k = tile if tile_k is None else tile_k
    nTq, nTk = num_tiles(grid, tile), num_tiles(grid_k, tile_k)
    if not 0 <= prefix <= nTk:
        raise ValueError(f"prefix must be in [0, {nTk}], got {prefix}")
    if not max(1, prefix) <= topk <= nTk:
        raise ValueError(f"topk must be in [{max(1, prefix)}, {nTk}], got {topk}")
    s = keep_prefix(tile_scores(pool(Q, grid, tile), pool(K, grid_k, tile_k)), prefix)
    idx = np.stack([topk_row(s[i], topk) for i in range(nTq)]).astype(np.int32)
    near = np.array([tie_gap(s[i], topk)[0] < NEAR_TIE_REL for i in range(nTq)])
    return idx, s, near


def select(q_bits, k_bits, grid, tile, topk: int, dtype: str = "bf16", grid_k=None, tile_k=None, prefix: int = 0):
    """All (b, h): idx [B, H, nTq, topk], scores [B, H, nTq, nTk], near_tie [B, H, nTq].

    q_bits [B, H, Nq, d] and k_bits [B, H, Nk, d] hold 16-bit patterns.
    """
    B, H = q_bits.shape[:2]
    nTq = num_tiles(grid, tile)
    nTk = num_tiles(grid if grid_k is None else grid_k, tile if tile_k is None else tile_k)
    idx = np.empty((B, H, nTq, topk), np.int32)
    sc = np.empty((B, H, nTq, nTk), np.float64)
    near = np.empty((B, H, nTq), bool)
    for b in range(B):
        for h in range(H):
            idx[b, h], sc[b, h], near[b, h] = select_head(
                widen(q_bits[b, h], dtype), widen(k_bits[b, h], dtype), grid, tile, topk, grid_k, tile_k, prefix)
    return idx, sc, near


def topk_from_sparsity(n_kv_tiles: int, sparsity: float, prefix: int = 0) -> int:
    """Kept blocks per query block for a sparsity in [0, 1): round((1 - s) * n), halves up,
    in [max(1, prefix), n]."""
    if not 0.0 <= sparsity < 1.0:
        raise ValueError(f"sparsity must be in [0, 1), got {sparsity}")
    k = math.floor((1.0 - sparsity) * n_kv_tiles + 0.5)
    return int(min(max(k, 1, prefix), n_kv_tiles))


def selection_is_valid(gpu_row: np.ndarray, s_row: np.ndarray, topk: int) -> bool:
    """Is a selection other than the oracle's still correct under a near-tie?

    It is when it has topk distinct ascending entries and every block in the
    symmetric difference with the oracle's list scores inside the band
    [s_(k+1) - delta, s_(k) + delta] around the cut.
    """
    nT = s_row.shape[0]
    g = np.asarray(gpu_row)
    if g.shape != (topk,) or np.any(g < 0) or np.any(g >= nT) or np.any(np.diff(g) <= 0):
        return False
    ref = topk_row(s_row, topk)
    diff = np.setxor1d(ref, g)
    if diff.size == 0:
        return True
    rel, delta = tie_gap(s_row, topk)
    if rel >= NEAR_TIE_REL:
        return False
    srt = np.sort(s_row)[::-1]
    lo, hi = srt[topk] - delta, srt[topk - 1] + delta
    return bool(np.all((s_row[diff] >= lo) & (s_row[diff] <= hi)))


# ------------------------------------------------------------------ attention
def attend_head(Q, K, V, grid, tile, idx, scale: float, query_tiles=None, grid_k=None, tile_k=None):
    """Block-sparse exact attention for one head.

    Q: [Nq, d], K, V: [Nk, d] float64 (K and V tiled with grid_k / tile_k,
    default the query's).  idx: [nTq, topk] kept key/value blocks per query
    block.  Returns O [Nq, d] and LSE [Nq]; rows of query blocks not in
    ``query_tiles`` (default: all) are NaN.
    """
    toks = tile_tokens(grid, tile)
    ktoks = tile_tokens(grid if grid_k is None else grid_k, tile if tile_k is None else tile_k)
    N, d = Q.shape
    O = np.full((N, V.shape[1]), np.nan)
    L = np.full(N, np.nan)
    tiles = range(len(toks)) if query_tiles is None else query_tiles
    for i in tiles:
        rows = toks[i]
        keys = np.concatenate([ktoks[j] for j in idx[i]])
        z = scale * (Q[rows] @ K[keys].T)
        m = z.max(axis=1, keepdims=True)
        e = np.exp(z - m)
        l = e.sum(axis=1, keepdims=True)
        O[rows] = (e @ V[keys]) / l
        L[rows] = (m + np.log(l))[:, 0]
    return O, L


def dense_bruteforce(Q, K, V, scale: float):
    """Dense softmax attention over all N tokens (no tiles): O [N, d], LSE [N]."""
    z = scale * (Q @ K.T)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ V) / l, (m + np.log(l))[:, 0]


# ----------------------------------------------------------- coarse branch
def coarse_head(Q, K, V, grid, tile, scale: float, grid_k=None, tile_k=None):
    """Tile-level attention of one head (docstring step 9): o_coarse [nTq, d].

    Q: [Nq, d], K, V: [Nk, d] float64; K and V pooled on grid_k / tile_k
    (default the query's)."""
    grid_k = grid if grid_k is None else grid_k
    tile_k = tile if tile_k is None else tile_k
    qbar, kbar, vbar = pool(Q, grid, tile), pool(K, grid_k, tile_k), pool(V, grid_k, tile_k)
    z = scale * tile_scores(qbar, kbar)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    return (e @ vbar) / e.sum(axis=1, keepdims=True)


def gated_output(O_sparse, gate, o_coarse, grid, tile):
    """O_sparse + gate * o_coarse of each token's query block (docstring step 9).

    O_sparse, gate: [Nq, d]; o_coarse: [nTq, d].  Returns a new [Nq, d] array."""
    out = np.array(O_sparse, dtype=np.float64, copy=True)
    for i, tok in enumerate(tile_tokens(grid, tile)):
        out[tok] += gate[tok] * o_coarse[i]
    return out
