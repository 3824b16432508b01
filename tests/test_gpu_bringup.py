"""Building blocks of the attend kernel on the GPU, each against a host
reference: the 5-D TMA box (tile index map, edge zero fill, 128-byte
swizzle), the shared-memory x shared-memory MMA (S = Q K^T) and the
TMEM x shared-memory MMA (O = P V)."""
import ctypes
import os

import numpy as np
import pytest
import torch

from block_sparse_video_tile_b200 import api, synth
from oracle import vsa_oracle as vo

pytestmark = pytest.mark.gpu

_PKG = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "block_sparse_video_tile_b200")


def _diag():
    L = ctypes.CDLL(os.path.join(_PKG, "libvsa_diag.so"))
    P = ctypes.c_void_p
    L.vsa_diag_tma_box.argtypes = [ctypes.c_void_p, P, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_int32, ctypes.c_int32, P, P]
    L.vsa_diag_mma_ss.argtypes = [P, P, ctypes.c_int32, P, P]
    L.vsa_diag_mma_ts.argtypes = [P, P, ctypes.c_int32, P, P]
    L.vsa_diag_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    return L


def _err(L):
    c = ctypes.c_uint32()
    assert L.vsa_diag_error(ctypes.byref(c)) == 0
    return c.value


def _rand_bits(shape, seed):
    rng = np.random.default_rng(seed)
    return synth.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


@pytest.mark.parametrize("d,grid,tile,box_t,j,toff", [
    (128, (9, 20, 20), (4, 8, 8), 2, 0, 0),      # interior half-tile
    (128, (9, 20, 20), (4, 8, 8), 2, 26, 0),     # corner tile: partial t, y, x
    (128, (9, 20, 20), (4, 8, 8), 2, 13, 2),     # second t-half
    (64, (6, 10, 14), (4, 4, 4), 4, 23, 0),      # 64-token tile at the far corner
])
def test_tma_box(d, grid, tile, box_t, j, toff):
    L = _diag()
    B, H = 1, 3
    bh = 2
    T, Hh, W = grid
    x = _rand_bits((B, H, T * Hh * W, d), 7)
    xd = torch.from_numpy(x).view(torch.bfloat16).cuda()
    rows = box_t * tile[1] * tile[2]
    out = torch.zeros(((d // 64) * rows * 128,), dtype=torch.uint8, device="cuda")
    shp = api.make_shape(B, H, grid, d, tile)
    assert L.vsa_diag_tma_box(ctypes.byref(shp), xd.data_ptr(), box_t, j, toff, bh, out.data_ptr(),
                              None) == 0
    assert _err(L) == 0
    got = out.cpu().numpy().view(np.uint16)
    nTt, nTy, nTx = vo.tiles_per_axis(grid, tile)
    bt, by, bx = j // (nTy * nTx), (j // nTx) % nTy, j % nTx
    t0, y0, x0 = bt * tile[0] + toff, by * tile[1], bx * tile[2]
    exp = np.zeros_like(got)
    for sl in range(d // 64):
        for r in range(rows):
            lt, ly, lx = r // (tile[1] * tile[2]), (r // tile[2]) % tile[1], r % tile[2]
            t, y, xx = t0 + lt, y0 + ly, x0 + lx
            for c in range(8):
                off = (sl * rows * 128 + r * 128 + ((c ^ (r & 7)) * 16)) // 2
                if t < T and y < Hh and xx < W:
                    n = (t * Hh + y) * W + xx
                    exp[off:off + 8] = x[0, bh, n, sl * 64 + 8 * c: sl * 64 + 8 * c + 8]
    np.testing.assert_array_equal(got, exp)


@pytest.mark.parametrize("d", [64, 128])
def test_mma_ss(d):
    L = _diag()
    a = _rand_bits((128, d), 1)
    b = _rand_bits((128, d), 2)
    C = torch.zeros((128, 128), dtype=torch.float32, device="cuda")
    ad, bd = (torch.from_numpy(x).view(torch.bfloat16).cuda() for x in (a, b))
    assert L.vsa_diag_mma_ss(ad.data_ptr(), bd.data_ptr(), d, C.data_ptr(), None) == 0
    assert _err(L) == 0
    ref = vo.bf16_to_f64(a) @ vo.bf16_to_f64(b).T
    np.testing.assert_allclose(C.cpu().numpy(), ref, rtol=0, atol=1e-4)


@pytest.mark.parametrize("d", [64, 128])
def test_mma_ts(d):
    L = _diag()
    p = _rand_bits((128, 128), 3)
    v = _rand_bits((128, d), 4)
    # two bf16 per 32-bit column, the lower key index in the low half
    packed = (p[:, 0::2].astype(np.uint32) | (p[:, 1::2].astype(np.uint32) << 16)).astype(np.uint32)
    pd = torch.from_numpy(packed.view(np.int32)).cuda()
    vd = torch.from_numpy(v).view(torch.bfloat16).cuda()
    O = torch.zeros((128, d), dtype=torch.float32, device="cuda")
    assert L.vsa_diag_mma_ts(pd.data_ptr(), vd.data_ptr(), d, O.data_ptr(), None) == 0
    assert _err(L) == 0
    ref = vo.bf16_to_f64(p) @ vo.bf16_to_f64(v)
    np.testing.assert_allclose(O.cpu().numpy(), ref, rtol=0, atol=1e-4)


def test_exp2_polynomial_vs_bounds():
    """The FMA-pipe 2^x of the softmax: relative error <= 8e-5 against the
    exact value on [-125, 8] (the fit reports 7.5e-5), exactly 0 below -125
    and at -inf; the multi-function-unit 2^x is checked on the same points."""
    L = _diag()
    L.vsa_diag_exp2.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int32, ctypes.c_void_p]
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125, 8, 200_001), rng.uniform(-30, 8, 100_000),
                        [-125.5, -200.0, -np.inf, 0.0, -0.0, 8.0, 0.5, -0.5]]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yp = torch.empty_like(xd)
    ym = torch.empty_like(xd)
    assert L.vsa_diag_exp2(xd.data_ptr(), yp.data_ptr(), ym.data_ptr(), x.size, None) == 0
    assert _err(L) == 0
    yp, ym = yp.cpu().numpy().astype(np.float64), ym.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    ok = x >= -125
    assert np.max(np.abs(yp[ok] - ref[ok]) / ref[ok]) <= 8e-5
    assert np.all(yp[~ok] == 0.0)
    assert np.max(np.abs(ym[ok] - ref[ok]) / ref[ok]) <= 1e-6


def test_bounded_wait_times_out_and_reports():
    """Failure detection without a GPU fault: a wait on a barrier that nothing
    arrives on gives up after its limit (1 s), the kernel returns, and the
    timeout code (1) is in the error word; the context stays usable."""
    L = _diag()
    L.vsa_diag_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.vsa_diag_wait_timeout(flag.data_ptr(), None) == 0
    assert _err(L) == 1
    assert int(flag.item()) == 1
    assert _err(L) == 0                       # read-and-clear
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0        # the context still works
