"""ctypes bindings of libvsa.so (declarations in include/vsa.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind these symbols.  Loading fails loudly when the library has not
been built -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvsa.so")

STATUS = {
    0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_TOPK_RANGE", 3: "VSA_ERR_UNSUPPORTED",
    4: "VSA_ERR_ALIGNMENT", 5: "VSA_ERR_WORKSPACE", 6: "VSA_ERR_ARCH", 7: "VSA_ERR_CUDA",
    8: "VSA_ERR_TOO_LARGE",
}
DEVERR = {0: "none", 1: "wait timeout", 2: "tile index out of range", 3: "kept list not strictly ascending"}

EXPORTS = ("vsa_tile_count", "vsa_kv_tile_count", "vsa_topk_from_sparsity", "vsa_select_workspace_bytes",
           "vsa_select", "vsa_select_noalloc", "vsa_attn_fwd", "vsa_select_coarse_workspace_bytes",
           "vsa_select_coarse", "vsa_attn_fwd_gated", "vsa_forward_host_workspace_bytes", "vsa_forward_host",
           "vsa_device_error", "vsa_status_string")
SELECT_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


DTYPE_BF16, DTYPE_F16 = 0, 1
LAYOUT_BHND, LAYOUT_BNHD = 0, 1


class VsaShape(ctypes.Structure):
    """vsa_shape: zero key/value fields mean "the query grid / tile"."""
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "T", "Hh", "W", "d", "tt", "th", "tw", "dtype", "layout",
                                              "Tk", "Hk", "Wk", "tk", "hk", "wk", "prefix_tiles")]


class VsaError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} failed: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_sparse_video_tile_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, S, I32, SZ = ctypes.c_void_p, ctypes.POINTER(VsaShape), ctypes.c_int32, ctypes.c_size_t
        L.vsa_tile_count.argtypes = [S, ctypes.POINTER(I32), ctypes.POINTER(I32)]
        L.vsa_tile_count.restype = ctypes.c_int
        L.vsa_kv_tile_count.argtypes = [S, ctypes.POINTER(I32), ctypes.POINTER(I32)]
        L.vsa_kv_tile_count.restype = ctypes.c_int
        L.vsa_topk_from_sparsity.argtypes = [S, ctypes.c_float, ctypes.POINTER(I32)]
        L.vsa_topk_from_sparsity.restype = ctypes.c_int
        L.vsa_select_workspace_bytes.argtypes = [S]
        L.vsa_select_workspace_bytes.restype = SZ
        L.vsa_select.argtypes = [S, P, P, I32, P, P, SZ, P]
        L.vsa_select.restype = ctypes.c_int
        L.vsa_select_noalloc.argtypes = [S, P, P, I32, P, P]
        L.vsa_select_noalloc.restype = ctypes.c_int
        L.vsa_attn_fwd.argtypes = [S, P, P, P, P, I32, ctypes.c_float, P, P, P]
        L.vsa_attn_fwd.restype = ctypes.c_int
        L.vsa_select_coarse_workspace_bytes.argtypes = [S]
        L.vsa_select_coarse_workspace_bytes.restype = SZ
        L.vsa_select_coarse.argtypes = [S, P, P, P, I32, ctypes.c_float, P, P, P, SZ, P]
        L.vsa_select_coarse.restype = ctypes.c_int
        L.vsa_attn_fwd_gated.argtypes = [S, P, P, P, P, I32, ctypes.c_float, P, P, P, P, P]
        L.vsa_attn_fwd_gated.restype = ctypes.c_int
        L.vsa_forward_host_workspace_bytes.argtypes = [S, I32, I32]
        L.vsa_forward_host_workspace_bytes.restype = SZ
        L.vsa_forward_host.argtypes = [S, P, P, P, I32, ctypes.c_float, P, P, P, I32, P, SZ, P]
        L.vsa_forward_host.restype = ctypes.c_int
        L.vsa_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), I32]
        L.vsa_device_error.restype = ctypes.c_int
        L.vsa_status_string.argtypes = [I32]
        L.vsa_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def check(call: str, status: int) -> None:
    if status != 0:
        raise VsaError(call, status)
