"""Python entry points over the C ABI, taking torch tensors.

PyTorch provides device memory and the current stream; the work is done by
libvsa's kernels.  Layouts (see include/vsa.h): Q, K, V, O bfloat16
[B, H, N, d] contiguous with raster token order over the latent grid (T, Hh, W);
idx int32 [B, H, nT, topk]; LSE float32 [B, H, N].
"""
from __future__ import annotations

import ctypes
import math

import torch

from ._native import VsaShape, check, lib

__all__ = ["make_shape", "tile_count", "select", "attn_fwd", "forward", "device_error",
           "select_workspace_bytes"]


def make_shape(B: int, H: int, grid, d: int, tile) -> VsaShape:
    T, Hh, W = grid
    tt, th, tw = tile
    return VsaShape(B, H, T, Hh, W, d, tt, th, tw)


def tile_count(grid, tile, d: int = 128, B: int = 1, H: int = 1):
    """(num_tiles, (tiles along T, Hh, W)) -- host only."""
    shp = make_shape(B, H, grid, d, tile)
    n = ctypes.c_int32()
    per = (ctypes.c_int32 * 3)()
    check("vsa_tile_count", lib().vsa_tile_count(ctypes.byref(shp), ctypes.byref(n), per))
    return n.value, (per[0], per[1], per[2])


def select_workspace_bytes(B, H, grid, d, tile) -> int:
    shp = make_shape(B, H, grid, d, tile)
    return int(lib().vsa_select_workspace_bytes(ctypes.byref(shp)))


def _check_qkv(name, x, B, H, N, d):
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor")
    if tuple(x.shape) != (B, H, N, d):
        raise ValueError(f"{name} has shape {tuple(x.shape)}, expected {(B, H, N, d)}")


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def select(q: torch.Tensor, k: torch.Tensor, grid, tile, topk: int, *, out=None,
           workspace=None, stream=None) -> torch.Tensor:
    """Top-k key tiles per query tile: int32 [B, H, nT, topk], ascending."""
    B, H, N, d = q.shape
    _check_qkv("q", q, B, H, N, d)
    _check_qkv("k", k, B, H, N, d)
    shp = make_shape(B, H, grid, d, tile)
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


def attn_fwd(q, k, v, idx, grid, tile, *, scale: float | None = None, out=None, lse=None,
             stream=None):
    """Block-sparse attention over the kept tiles: (O bf16 [B,H,N,d], LSE f32 [B,H,N])."""
    B, H, N, d = q.shape
    for name, x in (("q", q), ("k", k), ("v", v)):
        _check_qkv(name, x, B, H, N, d)
    if not (idx.is_cuda and idx.dtype == torch.int32 and idx.is_contiguous() and idx.dim() == 4):
        raise ValueError("idx must be a contiguous CUDA int32 tensor [B, H, nT, topk]")
    topk = idx.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    shp = make_shape(B, H, grid, d, tile)
    check("vsa_attn_fwd", lib().vsa_attn_fwd(
        ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), int(topk),
        float(scale), out.data_ptr(), lse.data_ptr(), _stream(stream)))
    return out, lse


def forward(q, k, v, grid, tile, topk: int, *, scale=None, stream=None):
    """select + attn_fwd: (O, LSE, idx)."""
    idx = select(q, k, grid, tile, topk, stream=stream)
    o, lse = attn_fwd(q, k, v, idx, grid, tile, scale=scale, stream=stream)
    return o, lse, idx


def device_error(reset: bool = True) -> int:
    """The kernels' device error word (0 = none); synchronizes the device."""
    code = ctypes.c_uint32()
    check("vsa_device_error", lib().vsa_device_error(ctypes.byref(code), 1 if reset else 0))
    return code.value
