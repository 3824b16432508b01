"""Ulysses-style sequence parallelism (block_sparse_video_tile_b200.seqpar) on
CPU: two and four gloo ranks, with the oracle standing in for the per-rank GPU
forward.  Checks that the two all-to-alls hand every rank the full sequence of
its heads and bring the output back to the right token slices, so that the
sharded forward equals the unsharded one head by head.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_video_tile_b200 import seqpar
from oracle import vsa_oracle as vo

CASES = {
    # name: (B, H, grid, tile, topk, grid_k, d)
    "self": (2, 4, (4, 4, 8), (2, 2, 4), 3, None, 8),
    "kv_grid": (1, 4, (4, 4, 8), (2, 2, 4), 4, (6, 4, 8), 8),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full(case):
    B, H, grid, tile, topk, grid_k, d = CASES[case]
    rng = np.random.default_rng(7)
    Nq, Nk = int(np.prod(grid)), int(np.prod(grid_k or grid))
    q = rng.standard_normal((B, Nq, H, d))
    k = rng.standard_normal((B, Nk, H, d))
    v = rng.standard_normal((B, Nk, H, d))
    return q, k, v


def _oracle_forward(q, k, v, grid, tile, topk, grid_k=None):
    """Per-head oracle forward of [B, N, h, d] float64 tensors: (O [B, N, h, d], LSE [B, h, N], idx)."""
    B, N, h, d = q.shape
    O = np.empty_like(q)
    L = np.empty((B, h, N))
    idxs = []
    for b in range(B):
        row = []
        for j in range(h):
            idx, _, _ = vo.select_head(q[b, :, j], k[b, :, j], grid, tile, topk, grid_k)
            O[b, :, j], L[b, j] = vo.attend_head(q[b, :, j], k[b, :, j], v[b, :, j], grid, tile, idx, d ** -0.5,
                                                 grid_k=grid_k)
            row.append(idx)
        idxs.append(row)
    return O, L, np.array(idxs)


def _attend(qh, kh, vh, grid, tile, topk, layout="bnhd", grid_k=None):
    assert layout == "bnhd"
    O, L, idx = _oracle_forward(qh.numpy(), kh.numpy(), vh.numpy(), grid, tile, topk, grid_k)
    return torch.from_numpy(O), torch.from_numpy(L), torch.from_numpy(idx)


def _worker(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, grid, tile, topk, grid_k, d = CASES[case]
        q, k, v = (torch.from_numpy(x) for x in _full(case))
        nq, nk = q.shape[1] // world, k.shape[1] // world
        mine = [x[:, rank * n:(rank + 1) * n].contiguous() for x, n in ((q, nq), (k, nk), (v, nk))]
        # round trip of the exchange alone
        back = seqpar.heads_to_seq(seqpar.seq_to_heads(mine[0]))
        rt = bool(torch.equal(back, mine[0]))
        # head shard = the full sequence of this rank's heads
        hs = seqpar.seq_to_heads(mine[1])
        h = H // world
        shard_ok = bool(torch.equal(hs, k[:, :, rank * h:(rank + 1) * h]))
        o, lse, idx = seqpar.forward_ulysses(*mine, grid, tile, topk, attend=_attend, grid_k=grid_k)
        out[rank] = (rt, shard_ok, o.numpy(), lse.numpy(), idx.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", sorted(CASES))
def test_ulysses_equals_unsharded(case, world):
    B, H, grid, tile, topk, grid_k, d = CASES[case]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), case, out), nprocs=world, join=True)
    q, k, v = _full(case)
    O, L, idx = _oracle_forward(q, k, v, grid, tile, topk, grid_k)
    nq, h = q.shape[1] // world, H // world
    for r in range(world):
        rt, shard_ok, o, lse, ix = out[r]
        assert rt and shard_ok
        np.testing.assert_array_equal(o, O[:, r * nq:(r + 1) * nq])           # exact: same arithmetic
        np.testing.assert_array_equal(lse, L[:, r * h:(r + 1) * h])
        np.testing.assert_array_equal(ix, idx[:, r * h:(r + 1) * h])


def test_divisibility_checked():
    import unittest.mock as um
    x = torch.zeros(1, 6, 3, 4)
    with um.patch.object(dist, "get_world_size", return_value=2):
        with pytest.raises(ValueError):
            seqpar.seq_to_heads(x)                 # 3 heads over 2 ranks
        with pytest.raises(ValueError):
            seqpar.heads_to_seq(torch.zeros(1, 7, 2, 4))   # 7 tokens over 2 ranks
