"""Seeded synthetic inputs for 3-D block-sparse video attention.

This module only draws numbers.  It holds none of the attention arithmetic
(no tiling, pooling, scoring, selection or softmax), so both the CUDA path and
the CPU oracle can take their inputs from it without sharing any of the
method.

Layout of every tensor it returns: ``[B, H, N, d]`` with the token index
``n = (t * Hh + y) * W + x`` (raster order over the post-patch latent grid
``(T, Hh, W)``), as ``uint16`` arrays holding bfloat16 bit patterns.

Two input families, matching the workloads the FastVideo VSA user guide and the
fastbsa page describe (video DiT attention over a latent grid):

* ``normal``:  Q, K, V i.i.d. N(0, 1), drawn in that order from one
  ``numpy.random.Generator(PCG64(seed))`` stream as float32, then rounded to
  bfloat16 (round to nearest even).
* ``field``:   Q and K share, per (batch, head, channel), a smooth
  low-frequency field over (t, y, x) -- a sum of 8 sinusoids with amplitude
  0.5, frequencies U(0, 1.5) cycles per grid extent on each axis and phase
  U(0, 2*pi) -- plus independent 0.5 * N(0, 1) noise each; V is N(0, 1).
  Neighbouring tiles therefore have related content, so tile selection is
  structured the way it is on real video latents.  Draw order: field
  parameters for all (b, h, c), then Q noise, then K noise, then V.
"""
from __future__ import annotations

import numpy as np

__all__ = ["f32_to_bf16_bits", "f32_to_f16_bits", "bf16_bits_to_f32", "make_qkv", "N_SINUSOIDS"]

N_SINUSOIDS = 8


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to IEEE half precision (nearest, ties to even); return the bits."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _field_params(rng: np.random.Generator, B: int, H: int, d: int):
    """Frequencies [B, H, d, 8, 3] (cycles per grid extent) and phases [B, H, d, 8]."""
    freq = rng.uniform(0.0, 1.5, size=(B, H, d, N_SINUSOIDS, 3))
    phase = rng.uniform(0.0, 2.0 * np.pi, size=(B, H, d, N_SINUSOIDS))
    return freq, phase


def _field_head(freq: np.ndarray, phase: np.ndarray, grid: tuple) -> np.ndarray:
    """Sum-of-sinusoids field of one head, float32 [N, d].

    Each sinusoid is 0.5 * sin(2*pi*(ft*t/T + fy*y/Hh + fx*x/W) + phi).  It is
    built as Im(0.5 e^{i phi} e^{i 2 pi ft t/T} * e^{i 2 pi (fy y/Hh + fx x/W)}),
    so the grid-sized sum is a batched complex matrix product with an inner
    dimension of 8 (one term per sinusoid).
    """
    T, Hh, W = grid
    d, S = phase.shape
    t = np.arange(T) / T
    y = np.arange(Hh) / Hh
    x = np.arange(W) / W
    et = np.exp(2j * np.pi * freq[:, :, 0, None] * t)                 # [d, S, T]
    et = et * (0.5 * np.exp(1j * phase))[:, :, None]
    ey = np.exp(2j * np.pi * freq[:, :, 1, None] * y)                 # [d, S, Hh]
    ex = np.exp(2j * np.pi * freq[:, :, 2, None] * x)                 # [d, S, W]
    eyx = (ey[:, :, :, None] * ex[:, :, None, :]).reshape(d, S, Hh * W)
    prod = np.matmul(et.transpose(0, 2, 1).astype(np.complex64), eyx.astype(np.complex64))
    return np.ascontiguousarray(prod.imag.reshape(d, T * Hh * W).T)


def make_qkv(B: int, H: int, grid: tuple, d: int, seed: int = 0,
             kind: str = "normal", dtype: str = "bf16", grid_k: tuple | None = None):
    """Return (q, k, v) as uint16 arrays holding bfloat16 bit patterns (dtype
    "bf16") or IEEE half-precision ones ("f16"): q [B, H, Nq, d] over ``grid``,
    k and v [B, H, Nk, d] over ``grid_k`` (default: the same grid).

    Values are drawn head by head in (b, h) order within each tensor; a
    Generator fills consecutive draws from one stream, so this equals drawing
    each whole tensor at once.  For structured inputs K's field is the same
    function of the normalised coordinates (t/T, y/Hh, x/W), sampled on its
    own grid.
    """
    grids = (grid, grid_k or grid, grid_k or grid)
    Ns = [g[0] * g[1] * g[2] for g in grids]
    rng = np.random.Generator(np.random.PCG64(seed))
    out = [np.empty((B, H, N, d), dtype=np.uint16) for N in Ns]
    to_bits = f32_to_f16_bits if dtype == "f16" else f32_to_bf16_bits
    if kind == "normal":
        for x, N in zip(out, Ns):
            for b in range(B):
                for h in range(H):
                    x[b, h] = to_bits(rng.standard_normal((N, d), dtype=np.float32))
        return tuple(out)
    if kind == "field":
        freq, phase = _field_params(rng, B, H, d)
        for x, g, N in zip(out[:2], grids[:2], Ns[:2]):   # the field is recomputed for K
            for b in range(B):
                for h in range(H):
                    fld = _field_head(freq[b, h], phase[b, h], g)
                    noise = rng.standard_normal((N, d), dtype=np.float32)
                    x[b, h] = to_bits(fld + np.float32(0.5) * noise)
        for b in range(B):
            for h in range(H):
                out[2][b, h] = to_bits(rng.standard_normal((Ns[2], d), dtype=np.float32))
        return tuple(out)
    raise ValueError(f"unknown input kind {kind!r}")
