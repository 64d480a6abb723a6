"""Guard bytes around every output buffer (a stand-in for a memory checker).

Each output of dispatch, combine and the rows next to them is a view into a
larger allocation whose leading and trailing guard bytes hold a fixed pattern;
after the kernels run the guards must be untouched.  The cases cover every
dispatch path (direct-rank, histogram with padding, one-CTA and tiled metadata,
bulk and register scatter) and a capacity smaller than the batch needs.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests._lib import bf16_to_dev, to_dev
from workloads import normal_bf16_rows, random_problem

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import combine_route_meta_b200 as moe

GUARD = 4096
PATTERN = 0x5A


class Guarded:
    """A device buffer of `shape` x `dtype` between two guard regions."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        size = GUARD + (n + 15) // 16 * 16 + GUARD
        self.back = torch.full((size,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.back[GUARD:GUARD + n].view(dtype).view(shape) if n else \
            torch.empty(shape, dtype=dtype, device="cuda")

    @property
    def ptr(self):
        return ctypes.c_void_p(self.back.data_ptr() + GUARD)

    def intact(self):
        b = self.back.cpu().numpy()
        return bool(np.all(b[:GUARD] == PATTERN) and np.all(b[GUARD + self.n:] == PATTERN))


def _dispatch_guarded(x, idx, w, E, R, fp8, pad, rows_cap=None):
    T, H = x.shape
    k = idx.shape[1]
    cfg = moe.make_config(H, k, E, R, fp8, pad)
    cap = moe.rows_capacity(cfg, T) if rows_cap is None else rows_cap
    g = dict(recv_x=Guarded((cap, H), torch.uint8 if fp8 else torch.int16),
             recv_scale=Guarded((cap, H // 128), torch.float32) if fp8 else None,
             count=Guarded((E,), torch.int32), offset=Guarded((E + 1,), torch.int32),
             rank=Guarded((R + 1,), torch.int32), src=Guarded((cap,), torch.int32),
             slot=Guarded((T, k), torch.int32),
             ws=Guarded((max(moe.workspace_bytes(cfg, T), 1),), torch.uint8))
    out = moe.moe_dispatch_out(g["recv_x"].ptr.value, g["recv_scale"].ptr.value if fp8 else None,
                               g["count"].ptr.value, g["offset"].ptr.value, g["rank"].ptr.value,
                               g["src"].ptr.value, cap)
    h = moe.moe_handle()
    err = moe.error_word()
    st = moe.moe_dispatch(ctypes.byref(cfg), T, ctypes.c_void_p(x.data_ptr()),
                          ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                          ctypes.byref(out), g["slot"].ptr, g["ws"].ptr, moe.workspace_bytes(cfg, T),
                          ctypes.c_void_p(err.data_ptr()), None, ctypes.byref(h))
    assert st == 0
    return g, h, cap


@pytest.mark.parametrize("T,H,E,R,k,fp8,pad,cap", [
    (128, 7168, 256, 8, 8, True, False, None),     # direct-rank decode kernel
    (256, 7168, 256, 32, 8, True, True, None),     # histogram kernel with padding
    (300, 1032, 16, 4, 5, False, False, None),     # one-CTA metadata, register scatter
    (600, 1024, 64, 8, 8, False, False, None),     # tiled metadata, bulk scatter
    (3000, 512, 256, 32, 8, True, True, None),     # tiled metadata, fp8 scatter, padding
    (100, 2048, 16, 4, 4, False, False, 250),      # capacity short of T*k: entries dropped
    (1500, 2048, 16, 4, 4, True, False, 3000),     # the same on the tiled path
])
def test_outputs_stay_inside_their_buffers(T, H, E, R, k, fp8, pad, cap):
    x, idx, w = random_problem(T + H, T, H, E, k)
    xd, idxd, wd = bf16_to_dev(x), to_dev(idx), to_dev(w)
    g, h, rows = _dispatch_guarded(xd, idxd, wd, E, R, fp8, pad, cap)
    # combine and the partial combine on the same handle
    eo = bf16_to_dev(normal_bf16_rows(3, 3, 0, rows, H))
    y = Guarded((T, H), torch.int16)
    assert moe.moe_combine(ctypes.byref(h), ctypes.c_void_p(eo.data_ptr()), y.ptr,
                           ctypes.c_void_p(moe.error_word().data_ptr()), None) == 0
    part, prank, npart, y2 = (Guarded((T, k, H), torch.int16), Guarded((T, k), torch.int32),
                              Guarded((T,), torch.int32), Guarded((T, H), torch.int16))
    assert moe.moe_combine_rank_partial(ctypes.byref(h), g["rank"].ptr, ctypes.c_void_p(eo.data_ptr()),
                                        part.ptr, prank.ptr, npart.ptr, y2.ptr,
                                        ctypes.c_void_p(moe.error_word().data_ptr()), None) == 0
    torch.cuda.synchronize()
    bits = moe.check()
    assert bits == (moe.DEV_CAPACITY if cap is not None else 0)
    for name, b in list(g.items()) + [("y", y), ("partial", part), ("prank", prank), ("npart", npart),
                                      ("y_partial", y2)]:
        if b is not None:
            assert b.intact(), name


@pytest.mark.parametrize("rows,I,in_use,col_major", [(1000, 2048, 990, False), (300, 384, 300, True)])
def test_silu_quant_stays_inside_its_buffers(rows, I, in_use, col_major):
    rng = np.random.default_rng(rows)
    gu = bf16_to_dev(normal_bf16_rows(5, 1, 0, rows, 2 * I))
    src = to_dev(np.where(rng.random(rows) < 0.1, -1, np.arange(rows)).astype(np.int32))
    act = Guarded((rows, I), torch.uint8)
    sc = Guarded((I // 128, rows) if col_major else (rows, I // 128), torch.float32)
    n = to_dev(np.array([in_use], np.int32))
    assert moe.moe_silu_quant(rows, I, ctypes.c_void_p(gu.data_ptr()), ctypes.c_void_p(src.data_ptr()),
                              ctypes.c_void_p(n.data_ptr()), act.ptr, sc.ptr, 1 if col_major else 0,
                              None) == 0
    torch.cuda.synchronize()
    assert act.intact() and sc.intact()


@pytest.mark.parametrize("T,E,k,G,TG", [(1000, 256, 8, 8, 4), (33, 1024, 32, 32, 2), (70, 96, 6, 4, 2)])
def test_router_stays_inside_its_buffers(T, E, k, G, TG):
    l = to_dev(np.random.default_rng(T).standard_normal((T, E)).astype(np.float32))
    idx, w = Guarded((T, k), torch.int32), Guarded((T, k), torch.float32)
    assert moe.moe_router_topk(T, E, k, ctypes.c_void_p(l.data_ptr()), moe.SCORE_SIGMOID, G, TG, 1,
                               idx.ptr, w.ptr, None) == 0
    torch.cuda.synchronize()
    assert idx.intact() and w.intact()
