"""vsa_select_noalloc against vsa_select, through the C ABI.

vsa_select_noalloc serves callers that cannot call cudaMalloc (a framework
that owns all device memory through its own pool, code in a region where
allocation is forbidden, a plugin without an allocator handle): it keeps the
pooled tile means in a fixed scratch array inside the library instead of a
caller-provided workspace.  Its indices must equal vsa_select's exactly, on
consecutive calls that reuse the shared scratch.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from block_sparse_video_tile_b200 import _native, api
from block_sparse_video_tile_b200.workloads import WAN5B, Workload
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

CASES = [
    Workload("ragged256", 1, 2, (9, 20, 20), 128, (4, 8, 8), 5),
    Workload("ragged64_d64", 1, 3, (5, 9, 11), 64, (4, 4, 4), 6),
    WAN5B,
]


def _select_with_workspace(shp, qd, kd, topk, out):
    ws = torch.empty(int(_native.lib().vsa_select_workspace_bytes(ctypes.byref(shp))),
                     dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    rc = _native.lib().vsa_select(ctypes.byref(shp), qd.data_ptr(), kd.data_ptr(), topk,
                                  out.data_ptr(), ws.data_ptr(), ws.numel(), st)
    assert rc == 0, _native.STATUS.get(rc, rc)


def _select_noalloc(shp, qd, kd, topk, out):
    st = torch.cuda.current_stream().cuda_stream
    rc = _native.lib().vsa_select_noalloc(ctypes.byref(shp), qd.data_ptr(), kd.data_ptr(), topk,
                                          out.data_ptr(), st)
    assert rc == 0, _native.STATUS.get(rc, rc)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_select(w):
    shp = api.make_shape(w.B, w.H, w.grid, w.d, w.tile)
    nT, _ = api.tile_count(w.grid, w.tile, w.d, w.B, w.H)
    for seed in (0, 1):                        # two calls in a row on the shared scratch
        _, (qd, kd, _vd) = gu.inputs(w, seed=seed)
        ref = torch.full((w.B, w.H, nT, w.topk), -1, dtype=torch.int32, device="cuda")
        got = torch.full_like(ref, -2)
        _select_with_workspace(shp, qd, kd, w.topk, ref)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _select_noalloc(shp, qd, kd, w.topk, got)
        torch.cuda.synchronize()
        # the scratch belongs to the loaded library: this call takes no device memory
        assert torch.cuda.mem_get_info()[0] == free_before, "vsa_select_noalloc allocated device memory"
        assert torch.equal(ref, got), f"seed {seed}: noalloc indices differ"
        assert int(ref.min()) >= 0
    gu.assert_no_device_error()
