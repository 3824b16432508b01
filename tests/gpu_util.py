"""Shared helpers of the GPU tests: upload synthetic inputs, run the library,
and compare against the oracle with the stated tolerances.

Tolerances (float64 oracle vs the bfloat16/float32 CUDA path), over valid
query tokens: O max-abs <= 2e-2 and mean-abs <= 2e-3; LSE abs <= 1e-3.
Selected tile indices must equal the oracle's, except rows whose k-th and
(k+1)-th oracle scores are within 1e-4 relative (near-ties), where any
selection inside the tie band is accepted and counted.
"""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_video_tile_b200 import api, synth
from oracle import vsa_oracle as vo

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def to_dev(bits: np.ndarray, dtype: str = "bf16") -> torch.Tensor:
    t = torch.float16 if dtype == "f16" else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(bits)).view(t).cuda()


_CACHE = {}


def inputs(w, seed=0):
    """((q, k, v) host 16-bit patterns [B, H, N, d], (q, k, v) device tensors
    in the workload's layout); the last two input sets are kept so that tests
    on the same workload do not redraw them."""
    key = (w.B, w.H, w.grid, w.grid_k, w.d, w.kind, seed, w.dtype)
    if key not in _CACHE:
        if len(_CACHE) >= 2:
            _CACHE.pop(next(iter(_CACHE)))
        _CACHE[key] = synth.make_qkv(w.B, w.H, w.grid, w.d, seed=seed, kind=w.kind, dtype=w.dtype,
                                     grid_k=w.grid_k)
    q, k, v = _CACHE[key]
    dev = [to_dev(x, w.dtype) for x in (q, k, v)]
    if w.layout == "bnhd":
        dev = [x.permute(0, 2, 1, 3).contiguous() for x in dev]
    return (q, k, v), tuple(dev)


def geo(w) -> dict:
    """Keyword arguments of api.attn_fwd for the workload's key/value grid and layout."""
    return dict(grid_k=w.grid_k, tile_k=w.tile_k, layout=w.layout)


def sel(w) -> dict:
    """Keyword arguments of api.select: geo(w) and the always-kept prefix tiles."""
    return dict(geo(w), prefix_tiles=w.prefix_tiles)


def to_bhnd(x: torch.Tensor, w) -> torch.Tensor:
    """A device output in the workload's layout, as [B, H, N, ...]."""
    return x.permute(0, 2, 1, 3) if w.layout == "bnhd" else x


def oracle_scores(q, k, w):
    """float64 tile scores [B, H, nTq, nTk] straight from the oracle's steps (always-kept
    prefix tiles at +inf, as the selection sees them)."""
    B, H = q.shape[:2]
    out = []
    for b in range(B):
        for h in range(H):
            Q, K = vo.widen(q[b, h], w.dtype), vo.widen(k[b, h], w.dtype)
            out.append(vo.keep_prefix(vo.tile_scores(vo.pool(Q, w.grid, w.tile), vo.pool(K, w.kv_grid, w.kv_tile)),
                                      w.prefix_tiles))
    return np.stack(out).reshape(B, H, *out[0].shape)


def check_selection(gidx: np.ndarray, scores: np.ndarray, topk: int):
    """Returns (rows, near_tie_rows_accepted); asserts every row is correct."""
    B, H, nT, _ = scores.shape
    assert gidx.shape == (B, H, nT, topk)
    ties = 0
    for b in range(B):
        for h in range(H):
            for i in range(nT):
                ref = vo.topk_row(scores[b, h, i], topk)
                if np.array_equal(ref, gidx[b, h, i]):
                    continue
                assert vo.selection_is_valid(gidx[b, h, i], scores[b, h, i], topk), (
                    f"row (b={b}, h={h}, i={i}): gpu {gidx[b, h, i].tolist()} vs oracle {ref.tolist()}")
                ties += 1
    return B * H * nT, ties


def check_attention(o_gpu, lse_gpu, q, k, v, w, idx, scale, tiles=None):
    """Compare the GPU's O/LSE with the oracle on (b, h, query tile) triples
    (all of them when ``tiles`` is None).  Returns (max_abs, mean_abs, lse_abs)."""
    B, H = q.shape[:2]
    toks = vo.tile_tokens(w.grid, w.tile)
    o_gpu = to_bhnd(o_gpu, w).float().cpu().numpy()
    lse_gpu = lse_gpu.cpu().numpy()
    errs, lerrs = [], []
    by_head = {}
    if tiles is None:
        tiles = [(b, h, i) for b in range(B) for h in range(H) for i in range(len(toks))]
    for b, h, i in tiles:
        by_head.setdefault((b, h), []).append(i)
    for (b, h), ts in by_head.items():
        Q, K, V = (vo.widen(x[b, h], w.dtype) for x in (q, k, v))
        O, L = vo.attend_head(Q, K, V, w.grid, w.tile, idx[b, h], scale, query_tiles=ts,
                              grid_k=w.kv_grid, tile_k=w.kv_tile)
        rows = np.concatenate([toks[i] for i in ts])
        errs.append(np.abs(o_gpu[b, h][rows] - O[rows]))
        lerrs.append(np.abs(lse_gpu[b, h][rows] - L[rows]))
    e = np.concatenate([x.reshape(-1) for x in errs])
    le = np.concatenate(lerrs)
    max_abs, mean_abs, lse_abs = float(e.max()), float(e.mean()), float(le.max())
    assert np.isfinite(e).all() and np.isfinite(le).all()
    assert max_abs <= O_MAX_ABS, f"O max-abs {max_abs}"
    assert mean_abs <= O_MEAN_ABS, f"O mean-abs {mean_abs}"
    assert lse_abs <= LSE_ABS, f"LSE abs {lse_abs}"
    return max_abs, mean_abs, lse_abs


def assert_no_device_error():
    code = api.device_error(reset=True)
    assert code == 0, f"device error word {code}"
