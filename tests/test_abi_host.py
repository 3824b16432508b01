"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and its host-side geometry and argument checks behave as documented.  No
kernel is launched here (every call returns before touching a device)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from block_sparse_video_tile_b200 import _native, api
from block_sparse_video_tile_b200.workloads import ALL
from oracle import vsa_oracle as vo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "vsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(vsa_\w+)\s*\(", src, flags=re.M))


def test_library_exports_every_declared_symbol():
    declared = _declared()
    assert declared == set(_native.EXPORTS)
    L = ctypes.CDLL(_native.LIB_PATH)
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings():
    for code, name in _native.STATUS.items():
        assert _native.lib().vsa_status_string(code).decode() == name
    assert _native.lib().vsa_status_string(999).decode() == "VSA_ERR_UNKNOWN"


def test_routing_log_tile_count():
    # FastVideo VSA user guide, "Wan top-k behavior": (31,22,40) with 4x8x8 -> 120
    n, per = api.tile_count((31, 22, 40), (4, 8, 8))
    assert (n, per) == (120, (8, 3, 5))


@pytest.mark.parametrize("name", sorted(ALL))
def test_tile_count_matches_oracle(name):
    w = ALL[name]
    n, per = api.tile_count(w.grid, w.tile, w.d, w.B, w.H)
    assert n == vo.num_tiles(w.grid, w.tile)
    assert per == vo.tiles_per_axis(w.grid, w.tile)
    # transposed float32 tile means [2, B*H, d, nT rounded up to 4]
    ldT = -(-n // 4) * 4
    assert api.select_workspace_bytes(w.B, w.H, w.grid, w.d, w.tile) == 4 * 2 * w.B * w.H * w.d * ldT


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 3), (dict(d=0), 1), (dict(tile=(3, 8, 8)), 3), (dict(tile=(1, 16, 16)), 3),
    (dict(tile=(4, 8, 16)), 3), (dict(grid=(0, 22, 40)), 1), (dict(tile=(8, 8, 8)), 3),
    (dict(dtype=torch.float32), 3), (dict(layout="bhdn"), 3),
    # key/value side: its own tile must hold as many tokens; a partial grid is invalid
    (dict(tile_k=(4, 4, 4)), 3), (dict(tile_k=(2, 8, 8)), 3), (dict(grid_k=(31, 0, 40)), 1),
    (dict(grid_k=(31, 22, 40), tile_k=(1, 16, 16)), 3),
])
def test_unsupported_shapes(kw, status):
    args = dict(B=1, H=1, grid=(31, 22, 40), d=128, tile=(4, 8, 8))
    args.update(kw)
    shp = api.make_shape(**args)
    n = ctypes.c_int32()
    assert _native.lib().vsa_tile_count(ctypes.byref(shp), ctypes.byref(n), None) == status
    assert _native.lib().vsa_select_workspace_bytes(ctypes.byref(shp)) == 0


def _sel(shp, q=256, k=512, topk=4, idx=1024, ws=2048, ws_bytes=1 << 30):
    return _native.lib().vsa_select(ctypes.byref(shp), q, k, topk, idx, ws, ws_bytes, None)


def _att(shp, q=256, k=512, v=768, idx=1024, topk=4, scale=0.1, o=2048, lse=4096):
    return _native.lib().vsa_attn_fwd(ctypes.byref(shp), q, k, v, idx, topk, scale, o, lse, None)


def test_argument_checks_before_launch():
    """Every one of these fails validation, so no device is ever touched."""
    shp = api.make_shape(1, 2, (31, 22, 40), 128, (4, 8, 8))
    assert _sel(shp, topk=0) == 2
    assert _sel(shp, topk=121) == 2
    assert _sel(shp, topk=-3) == 2
    assert _sel(shp, q=0) == 1
    assert _sel(shp, q=8) == 4                       # not 16-byte aligned
    assert _sel(shp, idx=2) == 4
    assert _sel(shp, ws=0) == 5
    assert _sel(shp, ws_bytes=16) == 5
    assert _att(shp, topk=0) == 2
    assert _att(shp, topk=121) == 2
    assert _att(shp, scale=0.0) == 1
    assert _att(shp, scale=float("nan")) == 1
    assert _att(shp, scale=float("inf")) == 1
    assert _att(shp, v=0) == 1
    assert _att(shp, o=24) == 4
    assert _att(shp, lse=6) == 4
    shp_bad = api.make_shape(1, 2, (31, 22, 40), 80, (4, 8, 8))
    assert _att(shp_bad) == 3
    assert _sel(shp_bad) == 3


def test_too_large_rejected():
    shp = api.make_shape(1, 1, (64, 64, 64), 128, (4, 4, 4))   # 4096 tiles
    n = ctypes.c_int32()
    assert _native.lib().vsa_tile_count(ctypes.byref(shp), ctypes.byref(n), None) == 8


def test_python_wrapper_raises():
    with pytest.raises(_native.VsaError) as e:
        api.tile_count((31, 22, 40), (3, 8, 8))
    assert e.value.status == 3


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """vsa_select_noalloc has a fixed scratch of 32 MiB: larger pooled-mean
    buffers are refused before any launch."""
    big = api.make_shape(8, 40, (18, 48, 80), 128, (4, 8, 8))     # 2*320*300*128*4 B = 98 MB
    small = api.make_shape(1, 24, (31, 22, 40), 128, (4, 8, 8))
    L = _native.lib()
    assert L.vsa_select_workspace_bytes(ctypes.byref(big)) > _native.SELECT_NOALLOC_SCRATCH_BYTES
    assert L.vsa_select_workspace_bytes(ctypes.byref(small)) <= _native.SELECT_NOALLOC_SCRATCH_BYTES
    assert L.vsa_select_noalloc(ctypes.byref(big), 256, 512, 4, 1024, None) == 5
    assert L.vsa_select_noalloc(ctypes.byref(small), 256, 512, 0, 1024, None) == 2
    assert L.vsa_select_noalloc(ctypes.byref(small), 8, 512, 4, 1024, None) == 4


def test_f16_shape_accepted():
    shp = api.make_shape(1, 2, (31, 22, 40), 128, (4, 8, 8), torch.float16)
    assert shp.dtype == _native.DTYPE_F16
    n = ctypes.c_int32()
    assert _native.lib().vsa_tile_count(ctypes.byref(shp), ctypes.byref(n), None) == 0 and n.value == 120


def test_kv_tile_count_and_workspace():
    # query: (31, 22, 40) / 4x8x8 -> 120 tiles; keys: (12, 48, 80) / 2x8x16 -> 6 * 6 * 5 = 180
    shp = api.make_shape(2, 3, (31, 22, 40), 64, (4, 8, 8), grid_k=(12, 48, 80), tile_k=(2, 8, 16))
    n, per = ctypes.c_int32(), (ctypes.c_int32 * 3)()
    assert _native.lib().vsa_tile_count(ctypes.byref(shp), ctypes.byref(n), per) == 0 and n.value == 120
    assert _native.lib().vsa_kv_tile_count(ctypes.byref(shp), ctypes.byref(n), per) == 0
    assert (n.value, tuple(per)) == (vo.num_tiles((12, 48, 80), (2, 8, 16)), (6, 6, 5))
    assert api.kv_tile_count((31, 22, 40), (4, 8, 8), (12, 48, 80), (2, 8, 16))[0] == 180
    # means: Q [B*H, d, 120] and K [B*H, d, 180] in float32
    assert api.select_workspace_bytes(2, 3, (31, 22, 40), 64, (4, 8, 8), (12, 48, 80), (2, 8, 16)) == \
        4 * 6 * 64 * (120 + 180)
    # without a key/value grid both sides are the query's
    shp0 = api.make_shape(1, 1, (12, 48, 80), 128, (4, 4, 4))
    assert _native.lib().vsa_kv_tile_count(ctypes.byref(shp0), ctypes.byref(n), None) == 0 and n.value == 720


@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.85, 0.9, 0.9375, 0.99, 0.999])
def test_topk_from_sparsity_matches_oracle(sparsity):
    for grid, tile, grid_k, tile_k in (((12, 48, 80), (4, 4, 4), None, None),
                                      ((31, 22, 40), (4, 8, 8), None, None),
                                      ((8, 16, 16), (4, 4, 4), (10, 20, 30), (2, 4, 8))):
        n = vo.num_tiles(grid_k or grid, tile_k or tile)
        assert api.topk_from_sparsity(grid, tile, sparsity, grid_k, tile_k) == vo.topk_from_sparsity(n, sparsity)


def test_topk_from_sparsity_range():
    for bad in (1.0, -0.01, float("nan")):
        with pytest.raises(_native.VsaError):
            api.topk_from_sparsity((12, 48, 80), (4, 4, 4), bad)


def test_bnhd_layout_and_kv_grid_accepted_on_host():
    shp = api.make_shape(2, 4, (9, 20, 20), 128, (4, 8, 8), torch.float16, layout="bnhd",
                         grid_k=(13, 16, 24), tile_k=(2, 8, 16))
    n = ctypes.c_int32()
    assert _native.lib().vsa_tile_count(ctypes.byref(shp), ctypes.byref(n), None) == 0 and n.value == 27
    assert _native.lib().vsa_kv_tile_count(ctypes.byref(shp), ctypes.byref(n), None) == 0
    assert n.value == vo.num_tiles((13, 16, 24), (2, 8, 16))


def test_prefix_tiles_checked_before_launch():
    # 120 tiles; prefix beyond them is invalid, topk below the prefix is out of range
    bad = api.make_shape(1, 2, (31, 22, 40), 128, (4, 8, 8), prefix_tiles=121)
    n = ctypes.c_int32()
    assert _native.lib().vsa_tile_count(ctypes.byref(bad), ctypes.byref(n), None) == 1
    shp = api.make_shape(1, 2, (31, 22, 40), 128, (4, 8, 8), prefix_tiles=15)
    assert _sel(shp, topk=14) == 2
    assert _native.lib().vsa_tile_count(ctypes.byref(shp), ctypes.byref(n), None) == 0
    assert api.topk_from_sparsity((31, 22, 40), (4, 8, 8), 0.99, prefix_tiles=15) == 15


def _selc(shp, q=256, k=512, v=768, topk=4, scale=0.1, idx=1024, coarse=2048, ws=4096, ws_bytes=1 << 30):
    return _native.lib().vsa_select_coarse(ctypes.byref(shp), q, k, v, topk, scale, idx, coarse, ws, ws_bytes, None)


def _attg(shp, coarse=8192, gate=16384, **kw):
    a = dict(q=256, k=512, v=768, idx=1024, topk=4, scale=0.1, o=2048, lse=4096)
    a.update(kw)
    return _native.lib().vsa_attn_fwd_gated(ctypes.byref(shp), a["q"], a["k"], a["v"], a["idx"], a["topk"],
                                            a["scale"], coarse, gate, a["o"], a["lse"], None)


def test_coarse_entry_points_check_arguments_before_launch():
    """The pooled coarse branch's calls validate like the others: no device is touched."""
    shp = api.make_shape(1, 2, (31, 22, 40), 128, (4, 8, 8))
    need = int(_native.lib().vsa_select_coarse_workspace_bytes(ctypes.byref(shp)))
    assert need == 4 * 2 * 128 * (120 + 2 * 120)            # Q, K and V means, float32
    assert _selc(shp, v=0) == 1
    assert _selc(shp, coarse=0) == 1
    assert _selc(shp, scale=0.0) == 1
    assert _selc(shp, topk=121) == 2
    assert _selc(shp, v=8) == 4
    assert _selc(shp, ws_bytes=need - 1) == 5
    assert _attg(shp, coarse=0) == 1                        # the gate needs its coarse output
    assert _attg(shp, gate=0) == 1
    assert _attg(shp, gate=24) == 4
    assert _attg(shp, coarse=8200) == 4
    assert _attg(shp, topk=0) == 2


def test_forward_host_checks_arguments_before_launch():
    shp = api.make_shape(1, 2, (31, 22, 40), 128, (4, 8, 8))
    L = _native.lib()
    need = int(L.vsa_forward_host_workspace_bytes(ctypes.byref(shp), 64, 2))
    assert need > 0 and need % 256 == 0
    assert int(L.vsa_forward_host_workspace_bytes(ctypes.byref(shp), 121, 2)) == 0
    args = [ctypes.byref(shp), 256, 512, 768, 64, 0.1, 1024, 2048, 4096, 2, 8192, need, None]
    def call(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return L.vsa_forward_host(*a)
    assert call(a1=0) == 1                     # q
    assert call(a5=0.0) == 1                   # scale
    assert call(a4=0) == 2                     # topk
    assert call(a10=8200) == 4                 # workspace alignment
    assert call(a11=need - 1) == 5             # workspace size
