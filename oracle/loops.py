"""Pure-Python loop restatement of the oracle, for tiny inputs only.

TEST INFRASTRUCTURE ONLY (imported by the tests alone).  It uses no NumPy
arithmetic and no code from ``vsa_oracle``: Python floats (IEEE double),
``math.exp``/``math.log`` and explicit loops, so that a mistake in the
vectorised oracle (a transposed operand, a wrong axis, a dropped token) shows
up as a disagreement between the two.

Steps follow the same reading of the pages as ``vsa_oracle`` (FastVideo VSA
user guide: blocks with ceil tiling, mean-pooled block scores, top-k kept
blocks per query block with ties to the lower index; exact softmax over the
kept blocks' tokens with scale head_size ** -0.5).
"""
from __future__ import annotations

import math


def _ceil_div(a, b):
    return (a + b - 1) // b


def blocks(grid, tile):
    """List of blocks in raster block order; each a list of (t, y, x) tokens."""
    T, Hh, W = grid
    tt, th, tw = tile
    out = []
    for bt in range(_ceil_div(T, tt)):
        for by in range(_ceil_div(Hh, th)):
            for bx in range(_ceil_div(W, tw)):
                toks = []
                for t in range(bt * tt, bt * tt + tt):
                    for y in range(by * th, by * th + th):
                        for x in range(bx * tw, bx * tw + tw):
                            if t < T and y < Hh and x < W:
                                toks.append((t, y, x))
                out.append(toks)
    return out


def _row(X, grid, tok):
    T, Hh, W = grid
    t, y, x = tok
    return X[(t * Hh + y) * W + x]


def mean_rows(X, grid, toks):
    d = len(X[0])
    acc = [0.0] * d
    for tok in toks:
        r = _row(X, grid, tok)
        for c in range(d):
            acc[c] += r[c]
    return [a / len(toks) for a in acc]


def dot(a, b):
    s = 0.0
    for u, v in zip(a, b):
        s += u * v
    return s


def select(Q, K, grid, tile, topk):
    """Q, K: lists of N rows (lists of floats).  Returns (idx, scores) per block."""
    bl = blocks(grid, tile)
    qb = [mean_rows(Q, grid, toks) for toks in bl]
    kb = [mean_rows(K, grid, toks) for toks in bl]
    nT = len(bl)
    scores = [[dot(qb[i], kb[j]) for j in range(nT)] for i in range(nT)]
    idx = []
    for i in range(nT):
        # rank of j = number of blocks that beat it (higher score, or equal and lower index)
        kept = []
        for j in range(nT):
            rank = 0
            for jj in range(nT):
                if scores[i][jj] > scores[i][j] or (scores[i][jj] == scores[i][j] and jj < j):
                    rank += 1
            if rank < topk:
                kept.append(j)
        idx.append(kept)
    return idx, scores


def attend(Q, K, V, grid, tile, idx, scale):
    """Returns O (dict token -> list) and LSE (dict token -> float) for every token."""
    bl = blocks(grid, tile)
    T, Hh, W = grid
    O, L = {}, {}
    for i, toks in enumerate(bl):
        keys = [tok for j in idx[i] for tok in bl[j]]
        for qt in toks:
            q = _row(Q, grid, qt)
            z = [scale * dot(q, _row(K, grid, kt)) for kt in keys]
            m = max(z)
            w = [math.exp(v - m) for v in z]
            l = sum(w)
            d = len(V[0])
            o = [0.0] * d
            for wk, kt in zip(w, keys):
                vr = _row(V, grid, kt)
                for c in range(d):
                    o[c] += wk * vr[c]
            n = (qt[0] * Hh + qt[1]) * W + qt[2]
            O[n] = [c / l for c in o]
            L[n] = m + math.log(l)
    return O, L


def coarse(Q, K, V, grid, tile, scale):
    """Tile-level attention: o_coarse per query block (list of lists)."""
    bl = blocks(grid, tile)
    qb = [mean_rows(Q, grid, toks) for toks in bl]
    kb = [mean_rows(K, grid, toks) for toks in bl]
    vb = [mean_rows(V, grid, toks) for toks in bl]
    out = []
    for i in range(len(bl)):
        z = [scale * dot(qb[i], kb[j]) for j in range(len(bl))]
        m = max(z)
        w = [math.exp(v - m) for v in z]
        l = sum(w)
        out.append([sum(w[j] * vb[j][c] for j in range(len(bl))) / l for c in range(len(vb[0]))])
    return out


def gated(O, G, oc, grid, tile):
    """O (dict or list by token) plus G[n] * oc[block of n], as a dict token -> list."""
    T, Hh, W = grid
    res = {}
    for i, toks in enumerate(blocks(grid, tile)):
        for t, y, x in toks:
            n = (t * Hh + y) * W + x
            res[n] = [O[n][c] + G[n][c] * oc[i][c] for c in range(len(oc[i]))]
    return res
