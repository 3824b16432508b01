"""Sequence-parallel (Ulysses-style) block-sparse attention over ranks.

FastVideo VSA user guide ("Verify routing and fallback"): the H3 route supports
pure Ulysses sequence parallelism and rejects ring or all-gather sequence
parallelism.  A DiT that keeps its activations sequence-sharded holds, on each
of P ranks, a contiguous slice of N/P tokens of every head.  Tile selection
needs all of a head's tiles and every query tile may keep any key tile, so a
head cannot be split along the sequence; instead one all-to-all turns the
sequence shards into head shards (each rank gets the full sequence of H/P
heads), each rank runs the block-sparse forward on its heads, and a second
all-to-all turns the output back into sequence shards.  The result is exactly
the unsharded forward of every head.

Tensors are token-major [B, N_local, H, d] (the [B, N, H, d] layout of the
library) with the rank's tokens contiguous: rank r holds tokens
r*N/P .. (r+1)*N/P - 1 of the raster order.  H and the token counts of the
query and key/value grids must be divisible by P.  The collectives are
torch.distributed all_to_all_single calls on the given process group (NCCL on
GPUs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api

__all__ = ["seq_to_heads", "heads_to_seq", "forward_ulysses"]


def _world(group) -> int:
    return dist.get_world_size(group)


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, N/P, H, d] sequence shard -> [B, N, H/P, d] head shard (rank r gets heads r*H/P ..)."""
    P = _world(group)
    B, n, H, d = x.shape
    if H % P:
        raise ValueError(f"heads ({H}) must be divisible by the group size ({P})")
    # [P (head group), B, n, H/P, d]: chunk p goes to rank p
    send = x.reshape(B, n, P, H // P, d).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[p] = rank p's token slice of my heads -> tokens in rank order
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * n, H // P, d).contiguous()


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """[B, N, H/P, d] head shard -> [B, N/P, H, d] sequence shard (the inverse of seq_to_heads)."""
    P = _world(group)
    B, N, h, d = y.shape
    if N % P:
        raise ValueError(f"tokens ({N}) must be divisible by the group size ({P})")
    n = N // P
    # [P (token slice), B, n, H/P, d]: slice p goes back to rank p
    send = y.reshape(B, P, n, h, d).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[p] = my token slice of rank p's heads -> heads in rank order
    return recv.permute(1, 2, 0, 3, 4).reshape(B, n, P * h, d).contiguous()


def forward_ulysses(q, k, v, grid, tile, topk=None, *, group=None, attend=None, **kw):
    """Block-sparse forward of sequence-sharded q, k, v ([B, N/P, H, d] each).

    Returns (O [B, N/P, H, d] sequence-sharded like q, LSE [B, H/P, Nq] and
    idx [B, H/P, nTq, topk] of this rank's heads).  ``attend`` is the per-rank
    forward (default ``api.forward``, called with layout="bnhd" and the
    remaining keyword arguments: sparsity, grid_k, tile_k, prefix_tiles, ...).
    """
    attend = api.forward if attend is None else attend
    qh, kh, vh = (seq_to_heads(x, group) for x in (q, k, v))
    o, lse, idx = attend(qh, kh, vh, grid, tile, topk, layout="bnhd", **kw)
    return heads_to_seq(o, group), lse, idx
