"""seqpar.forward_ulysses on one GPU: a one-rank NCCL group, so both
all-to-alls go through NCCL (as identity exchanges) around the CUDA forward;
the result must be bit-identical to calling the forward directly, and match
the float64 oracle (selection and attention of every head)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

from block_sparse_video_tile_b200 import api, seqpar
from block_sparse_video_tile_b200.workloads import Workload
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_equals_direct():
    w = Workload("seqpar1", 1, 4, (8, 12, 16), 128, (4, 4, 4), 6, "field", layout="bnhd", grid_k=(12, 12, 16),
                 prefix_tiles=12)
    (q, k, v), (qd, kd, vd) = gu.inputs(w, seed=5)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        topk = 14
        o, lse, idx = seqpar.forward_ulysses(qd, kd, vd, w.grid, w.tile, topk, grid_k=w.grid_k,
                                             prefix_tiles=w.prefix_tiles)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o2, lse2, idx2 = api.forward(qd, kd, vd, w.grid, w.tile, topk, grid_k=w.grid_k, layout="bnhd",
                                 prefix_tiles=w.prefix_tiles)
    gu.assert_no_device_error()
    assert torch.equal(idx, idx2) and torch.equal(o, o2) and torch.equal(lse, lse2)
    assert (idx[..., :w.prefix_tiles].cpu() == torch.arange(w.prefix_tiles)).all()
    wt = w.with_(topk=topk)
    gi = idx.cpu().numpy()
    gu.check_selection(gi, gu.oracle_scores(q, k, wt), topk)
    gu.check_attention(o, lse, q, k, v, wt, gi, w.d ** -0.5)
