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
           "forward", "forward_host", "device_error", "select_workspace_bytes"]


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


class _HostPipeline:
    """Device buffers, streams and events reused by forward_host for one shape."""

    def __init__(self, chunk, N, d, nT, topk, device, ws_bytes, dtype):
        mk = lambda *shape, dt=dtype: [torch.empty(shape, dtype=dt, device=device) for _ in range(2)]
        self.q, self.k, self.v, self.o = (mk(1, chunk, N, d) for _ in range(4))
        self.lse = mk(1, chunk, N, dt=torch.float32)
        self.idx = mk(1, chunk, nT, topk, dt=torch.int32)
        self.ws = [torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device) for _ in range(2)]
        self.s_in = torch.cuda.Stream(device)
        self.s_comp = torch.cuda.Stream(device)
        self.s_out = torch.cuda.Stream(device)
        self.key = (chunk, N, d, nT, topk, device, dtype)


_PIPE = {}


def forward_host(q, k, v, grid, tile, topk: int, *, scale=None, chunk_heads: int = 2,
                 out=None, lse=None, idx=None, device=None):
    """Host-to-host forward: select + attention for pinned CPU tensors.

    q, k, v: pinned CPU bfloat16 [B, H, N, d].  Returns (O, LSE, idx) in pinned
    CPU tensors (allocated unless given).  The (batch, head) pairs are
    processed in chunks of ``chunk_heads``: the upload of chunk c+1 and the
    download of chunk c-1 overlap the kernels of chunk c (three streams,
    double-buffered device memory).  Every chunk is one vsa_select and one
    vsa_attn_fwd call with H = chunk.  The caller's current stream waits for
    all of it, so work queued on it afterwards sees the outputs.
    """
    B, H, N, d = q.shape
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    for name, x in (("q", q), ("k", k), ("v", v)):
        if x.is_cuda or x.dtype != q.dtype or q.dtype not in _DTYPES or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU bfloat16/float16 tensor like q "
                             "(pinned for overlap)")
    nT, _ = tile_count(grid, tile, d, B, H)
    BH = B * H
    chunk = max(1, min(chunk_heads, BH))
    if out is None:
        out = torch.empty((B, H, N, d), dtype=q.dtype).pin_memory()
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    if idx is None:
        idx = torch.empty((B, H, nT, topk), dtype=torch.int32).pin_memory()
    key = (chunk, N, d, nT, topk, device, q.dtype)
    pipe = _PIPE.get(key)
    if pipe is None:
        pipe = _HostPipeline(chunk, N, d, nT, topk, device, select_workspace_bytes(1, chunk, grid, d, tile),
                             q.dtype)
        _PIPE.clear()
        _PIPE[key] = pipe
    caller = torch.cuda.current_stream(device)
    for s_ in (pipe.s_in, pipe.s_comp, pipe.s_out):
        s_.wait_stream(caller)
    qf, kf, vf = (x.view(BH, N, d) for x in (q, k, v))
    of, lf, xf = out.view(BH, N, d), lse.view(BH, N), idx.view(BH, nT, topk)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [None, None]
    for c, h0 in enumerate(range(0, BH, chunk)):
        nh = min(chunk, BH - h0)
        b = c % 2
        dq, dk, dv, do = (t[b][:, :nh] for t in (pipe.q, pipe.k, pipe.v, pipe.o))
        dl, di = pipe.lse[b][:, :nh], pipe.idx[b][:, :nh]
        with torch.cuda.stream(pipe.s_in):
            if ev_out[b] is not None:          # buffer b's previous outputs are downloaded
                pipe.s_in.wait_event(ev_out[b])
            dq.copy_(qf[h0:h0 + nh].unsqueeze(0), non_blocking=True)
            dk.copy_(kf[h0:h0 + nh].unsqueeze(0), non_blocking=True)
            dv.copy_(vf[h0:h0 + nh].unsqueeze(0), non_blocking=True)
            ev_in[b].record(pipe.s_in)
        with torch.cuda.stream(pipe.s_comp):
            pipe.s_comp.wait_event(ev_in[b])
            select(dq, dk, grid, tile, topk, out=di, workspace=pipe.ws[b], stream=pipe.s_comp)
            attn_fwd(dq, dk, dv, di, grid, tile, scale=scale, out=do, lse=dl, stream=pipe.s_comp)
            ev_comp[b].record(pipe.s_comp)
        with torch.cuda.stream(pipe.s_out):
            pipe.s_out.wait_event(ev_comp[b])
            of[h0:h0 + nh].unsqueeze(0).copy_(do, non_blocking=True)
            lf[h0:h0 + nh].unsqueeze(0).copy_(dl, non_blocking=True)
            xf[h0:h0 + nh].unsqueeze(0).copy_(di, non_blocking=True)
            e = torch.cuda.Event()
            e.record(pipe.s_out)
            ev_out[b] = e
    for s_ in (pipe.s_in, pipe.s_comp, pipe.s_out):
        caller.wait_stream(s_)
    return out, lse, idx


def device_error(reset: bool = True) -> int:
    """The kernels' device error word (0 = none); synchronizes the device."""
    code = ctypes.c_uint32()
    check("vsa_device_error", lib().vsa_device_error(ctypes.byref(code), 1 if reset else 0))
    return code.value
