"""Python entry points over the C ABI, taking torch tensors.

PyTorch provides device memory and the current stream; the work is done by
libvsa's kernels.  Layouts (see include/vsa.h): Q, K, V, O bfloat16 or float16,
contiguous, either "bhnd" = [B, H, N, d] or "bnhd" = [B, N, H, d], with raster
token order over the latent grid (T, Hh, W); idx int32 [B, H, nTq, topk];
LSE float32 [B, H, Nq].  Keys and values may have their own grid and tile
(grid_k, tile_k; by default the query's) with the same tile volume.
"""
from __future__ import annotations

import ctypes
import math

import torch

from ._native import DTYPE_BF16, DTYPE_F16, LAYOUT_BHND, LAYOUT_BNHD, VsaShape, check, lib

__all__ = ["make_shape", "tile_count", "kv_tile_count", "topk_from_sparsity", "select", "select_coarse", "attn_fwd",
           "forward", "forward_host", "device_error", "select_workspace_bytes", "select_coarse_workspace_bytes"]


_DTYPES = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}
_LAYOUTS = {"bhnd": LAYOUT_BHND, "bnhd": LAYOUT_BNHD}


def make_shape(B: int, H: int, grid, d: int, tile, dtype=torch.bfloat16, *, layout: str = "bhnd",
               grid_k=None, tile_k=None, prefix_tiles: int = 0) -> VsaShape:
    T, Hh, W = grid
    tt, th, tw = tile
    Tk, Hk, Wk = grid_k if grid_k is not None else (0, 0, 0)
    tk, hk, wk = tile_k if tile_k is not None else (0, 0, 0)
    return VsaShape(B, H, T, Hh, W, d, tt, th, tw, _DTYPES.get(dtype, -1), _LAYOUTS.get(layout, -1),
                    Tk, Hk, Wk, tk, hk, wk, prefix_tiles)


def _count(fn, shp):
    n = ctypes.c_int32()
    per = (ctypes.c_int32 * 3)()
    check(fn, getattr(lib(), fn)(ctypes.byref(shp), ctypes.byref(n), per))
    return n.value, (per[0], per[1], per[2])


def tile_count(grid, tile, d: int = 128, B: int = 1, H: int = 1):
    """(num query tiles, (tiles along T, Hh, W)) -- host only."""
    return _count("vsa_tile_count", make_shape(B, H, grid, d, tile))


def kv_tile_count(grid, tile, grid_k=None, tile_k=None, d: int = 128, B: int = 1, H: int = 1):
    """(num key/value tiles, (tiles along T, Hh, W)) -- host only."""
    return _count("vsa_kv_tile_count", make_shape(B, H, grid, d, tile, grid_k=grid_k, tile_k=tile_k))


def topk_from_sparsity(grid, tile, sparsity: float, grid_k=None, tile_k=None, d: int = 128,
                       prefix_tiles: int = 0) -> int:
    """Kept key/value tiles per query tile for a sparsity: round((1 - sparsity) * nTk), in
    [max(1, prefix_tiles), nTk]."""
    shp = make_shape(1, 1, grid, d, tile, grid_k=grid_k, tile_k=tile_k, prefix_tiles=prefix_tiles)
    k = ctypes.c_int32()
    check("vsa_topk_from_sparsity", lib().vsa_topk_from_sparsity(ctypes.byref(shp), float(sparsity),
                                                                  ctypes.byref(k)))
    return k.value


def select_workspace_bytes(B, H, grid, d, tile, grid_k=None, tile_k=None) -> int:
    shp = make_shape(B, H, grid, d, tile, grid_k=grid_k, tile_k=tile_k)
    return int(lib().vsa_select_workspace_bytes(ctypes.byref(shp)))


def select_coarse_workspace_bytes(B, H, grid, d, tile, grid_k=None, tile_k=None) -> int:
    shp = make_shape(B, H, grid, d, tile, grid_k=grid_k, tile_k=tile_k)
    return int(lib().vsa_select_coarse_workspace_bytes(ctypes.byref(shp)))


def _dims(x, layout):
    """(B, H, N, d) of a tensor in the given layout."""
    if x.dim() != 4:
        raise ValueError(f"expected a 4-D tensor, got shape {tuple(x.shape)}")
    if layout == "bhnd":
        return tuple(x.shape)
    if layout == "bnhd":
        B, N, H, d = x.shape
        return B, H, N, d
    raise ValueError(f"layout must be 'bhnd' or 'bnhd', got {layout!r}")


def _check_qkv(name, x, want, layout, dtype=None):
    if not (x.is_cuda and x.dtype in _DTYPES and x.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA bfloat16 or float16 tensor")
    if dtype is not None and x.dtype != dtype:
        raise ValueError(f"{name} is {x.dtype}, expected {dtype} like q")
    got = _dims(x, layout)
    if got != tuple(want):
        raise ValueError(f"{name} has (B, H, N, d) = {got} in layout {layout}, expected {tuple(want)}")


def _grid_tokens(grid) -> int:
    return grid[0] * grid[1] * grid[2]


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def select(q: torch.Tensor, k: torch.Tensor, grid, tile, topk: int, *, grid_k=None, tile_k=None,
           layout: str = "bhnd", prefix_tiles: int = 0, out=None, workspace=None, stream=None) -> torch.Tensor:
    """Top-k key tiles per query tile: int32 [B, H, nTq, topk], ascending; key/value
    tiles 0 .. prefix_tiles-1 are in every row (and count toward topk)."""
    B, H, Nq, d = _dims(q, layout)
    Nk = _grid_tokens(grid_k if grid_k is not None else grid)
    _check_qkv("q", q, (B, H, _grid_tokens(grid), d), layout)
    _check_qkv("k", k, (B, H, Nk, d), layout, q.dtype)
    shp = make_shape(B, H, grid, d, tile, q.dtype, layout=layout, grid_k=grid_k, tile_k=tile_k,
                     prefix_tiles=prefix_tiles)
    nT, _ = tile_count(grid, tile, d, B, H)
    if out is None:
        out = torch.empty((B, H, nT, topk), dtype=torch.int32, device=q.device)
    ws_bytes = int(lib().vsa_select_workspace_bytes(ctypes.byref(shp)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    check("vsa_select", lib().vsa_select(
        ctypes.byref(shp), q.data_ptr(), k.data_ptr(), int(topk), out.data_ptr(),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def select_coarse(q, k, v, grid, tile, topk: int, *, scale: float | None = None, grid_k=None, tile_k=None,
                  layout: str = "bhnd", prefix_tiles: int = 0, out=None, coarse=None, workspace=None, stream=None):
    """select() plus the pooled coarse branch: (idx, o_coarse f32 [B, H, nTq, d]),
    o_coarse[i] = sum_j softmax_j(scale * mean_i(Q) . mean_j(K)) mean_j(V)."""
    B, H, Nq, d = _dims(q, layout)
    Nk = _grid_tokens(grid_k if grid_k is not None else grid)
    _check_qkv("q", q, (B, H, _grid_tokens(grid), d), layout)
    for name, x in (("k", k), ("v", v)):
        _check_qkv(name, x, (B, H, Nk, d), layout, q.dtype)
    shp = make_shape(B, H, grid, d, tile, q.dtype, layout=layout, grid_k=grid_k, tile_k=tile_k,
                     prefix_tiles=prefix_tiles)
    nT, _ = tile_count(grid, tile, d, B, H)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, nT, topk), dtype=torch.int32, device=q.device)
    if coarse is None:
        coarse = torch.empty((B, H, nT, d), dtype=torch.float32, device=q.device)
    ws_bytes = int(lib().vsa_select_coarse_workspace_bytes(ctypes.byref(shp)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    check("vsa_select_coarse", lib().vsa_select_coarse(
        ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), int(topk), float(scale), out.data_ptr(),
        coarse.data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, coarse


def attn_fwd(q, k, v, idx, grid, tile, *, grid_k=None, tile_k=None, layout: str = "bhnd",
             scale: float | None = None, out=None, lse=None, coarse=None, gate=None, stream=None):
    """Block-sparse attention over the kept tiles: (O like q, LSE f32 [B, H, Nq]).
    With coarse (f32 [B, H, nTq, d], from select_coarse) and gate (like q), O
    also carries the gated coarse branch: O += gate * coarse[query tile]."""
    B, H, Nq, d = _dims(q, layout)
    Nk = _grid_tokens(grid_k if grid_k is not None else grid)
    _check_qkv("q", q, (B, H, _grid_tokens(grid), d), layout)
    for name, x in (("k", k), ("v", v)):
        _check_qkv(name, x, (B, H, Nk, d), layout, q.dtype)
    if not (idx.is_cuda and idx.dtype == torch.int32 and idx.is_contiguous() and idx.dim() == 4):
        raise ValueError("idx must be a contiguous CUDA int32 tensor [B, H, nTq, topk]")
    topk = idx.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    shp = make_shape(B, H, grid, d, tile, q.dtype, layout=layout, grid_k=grid_k, tile_k=tile_k)
    if out.dtype != q.dtype:
        raise ValueError("out must have the dtype of q")
    if (coarse is None) != (gate is None):
        raise ValueError("give both coarse and gate, or neither")
    if gate is None:
        check("vsa_attn_fwd", lib().vsa_attn_fwd(
            ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), int(topk),
            float(scale), out.data_ptr(), lse.data_ptr(), _stream(stream)))
        return out, lse
    _check_qkv("gate", gate, (B, H, Nq, d), layout, q.dtype)
    nT = idx.shape[2]
    if not (coarse.is_cuda and coarse.dtype == torch.float32 and coarse.is_contiguous()
            and tuple(coarse.shape) == (B, H, nT, d)):
        raise ValueError(f"coarse must be a contiguous CUDA float32 tensor of shape {(B, H, nT, d)}")
    check("vsa_attn_fwd_gated", lib().vsa_attn_fwd_gated(
        ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), int(topk),
        float(scale), coarse.data_ptr(), gate.data_ptr(), out.data_ptr(), lse.data_ptr(), _stream(stream)))
    return out, lse


def forward(q, k, v, grid, tile, topk: int | None = None, *, sparsity: float | None = None, grid_k=None,
            tile_k=None, layout: str = "bhnd", prefix_tiles: int = 0, scale=None, gate=None, stream=None):
    """select + attn_fwd: (O, LSE, idx).  Give topk, or sparsity (the fraction
    of key/value tiles left out, as in the fastbsa page's "Use" example).
    With gate (like q), O also carries the gated pooled coarse branch."""
    if (topk is None) == (sparsity is None):
        raise ValueError("give exactly one of topk and sparsity")
    if topk is None:
        topk = topk_from_sparsity(grid, tile, sparsity, grid_k, tile_k, _dims(q, layout)[3], prefix_tiles)
    kw = dict(grid_k=grid_k, tile_k=tile_k, layout=layout, stream=stream)
    if gate is None:
        idx = select(q, k, grid, tile, topk, prefix_tiles=prefix_tiles, **kw)
        o, lse = attn_fwd(q, k, v, idx, grid, tile, scale=scale, **kw)
    else:
        idx, coarse = select_coarse(q, k, v, grid, tile, topk, scale=scale, prefix_tiles=prefix_tiles, **kw)
        o, lse = attn_fwd(q, k, v, idx, grid, tile, scale=scale, coarse=coarse, gate=gate, **kw)
    return o, lse, idx


_HOST_WS = {}


def forward_host(q, k, v, grid, tile, topk: int, *, scale=None, chunk_heads: int = 2, grid_k=None, tile_k=None,
                 layout: str = "bhnd", prefix_tiles: int = 0, out=None, lse=None, idx=None, device=None,
                 stream=None):
    """Host-to-host forward through vsa_forward_host: select + attention for CPU tensors.

    q, k, v: CPU bfloat16/float16 tensors in ``layout`` (pinned for the copies
    to overlap the kernels).  Returns (O, LSE, idx) in CPU tensors (pinned,
    allocated unless given), complete when the call returns.  The (batch,
    head) pairs go through the GPU in chunks of ``chunk_heads`` heads,
    uploads and downloads overlapping the kernels (streams of the library);
    the device workspace is allocated here once per shape and reused.
    """
    B, H, Nq, d = _dims(q, layout)
    Nk = _grid_tokens(grid_k if grid_k is not None else grid)
    for name, x, n in (("q", q, Nq), ("k", k, Nk), ("v", v, Nk)):
        if x.is_cuda or x.dtype != q.dtype or q.dtype not in _DTYPES or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU bfloat16/float16 tensor like q "
                             "(pinned for overlap)")
        if _dims(x, layout) != (B, H, n, d):
            raise ValueError(f"{name} has (B, H, N, d) = {_dims(x, layout)}, expected {(B, H, n, d)}")
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    shp = make_shape(B, H, grid, d, tile, q.dtype, layout=layout, grid_k=grid_k, tile_k=tile_k,
                     prefix_tiles=prefix_tiles)
    nT, _ = tile_count(grid, tile, d, B, H)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32).pin_memory()
    if idx is None:
        idx = torch.empty((B, H, nT, topk), dtype=torch.int32).pin_memory()
    ws_bytes = int(lib().vsa_forward_host_workspace_bytes(ctypes.byref(shp), int(topk), int(chunk_heads)))
    if ws_bytes == 0:
        raise ValueError("invalid shape or topk")
    key = (device, ws_bytes)
    ws = _HOST_WS.get(key)
    if ws is None:
        _HOST_WS.clear()
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
        _HOST_WS[key] = ws
    st = torch.cuda.current_stream(device) if stream is None else stream
    check("vsa_forward_host", lib().vsa_forward_host(
        ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), int(topk), float(scale), out.data_ptr(),
        lse.data_ptr(), idx.data_ptr(), int(chunk_heads), ws.data_ptr(), ws_bytes, st.cuda_stream))
    st.synchronize()
    return out, lse, idx


def device_error(reset: bool = True) -> int:
    """The kernels' device error word (0 = none); synchronizes the device."""
    code = ctypes.c_uint32()
    check("vsa_device_error", lib().vsa_device_error(ctypes.byref(code), 1 if reset else 0))
    return code.value
