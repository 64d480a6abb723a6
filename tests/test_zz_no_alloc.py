"""moe_dispatch_no_alloc: the dispatch entry point for callers that cannot allocate.

Code that runs during CUDA graph capture, serving loops whose device memory is
planned once at start-up, and C hosts that only receive device pointers cannot
hand moe_dispatch a freshly allocated workspace.  The no-allocation entry point
keeps its metadata scratch in a fixed array inside the library instead.  This
test calls it through the C ABI and checks that it gives exactly what
moe_dispatch gives (dispatch results are compared bit for bit, as everywhere
in these tests), on two calls in a row with different inputs, so a second call
that finds the first call's scratch contents still gets the right answer.
It runs alone or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests._lib import bf16_from_dev, bf16_to_dev, to_dev
from workloads import random_problem

pytestmark = pytest.mark.gpu


def _dispatch(moe, entry, x, idx, w, E, R, fp8, pad128):
    """Runs one dispatch entry point on fresh buffers; returns host copies of all outputs."""
    T, H = x.shape
    k = idx.shape[1]
    cfg = moe.make_config(H, k, E, R, fp8, pad128)
    buf = moe.Buffers(cfg, T, "cuda")
    buf.recv_x.view(torch.uint8).fill_(0xA5)
    if buf.recv_scale is not None:
        buf.recv_scale.view(torch.uint8).fill_(0xA5)
    xd, idd, wd = bf16_to_dev(x), to_dev(idx), to_dev(w)
    moe.check()
    P = ctypes.c_void_p
    stream = P(torch.cuda.current_stream().cuda_stream)
    if entry == "moe_dispatch":
        st = moe.moe_dispatch(ctypes.byref(cfg), T, P(xd.data_ptr()), P(idd.data_ptr()),
                              P(wd.data_ptr()), ctypes.byref(buf.out), P(buf.slot.data_ptr()),
                              P(buf.workspace.data_ptr()), buf.workspace_bytes,
                              P(buf.err.data_ptr()), stream, ctypes.byref(buf.handle_c))
    else:
        st = moe.moe_dispatch_no_alloc(ctypes.byref(cfg), T, P(xd.data_ptr()), P(idd.data_ptr()),
                                       P(wd.data_ptr()), ctypes.byref(buf.out),
                                       P(buf.slot.data_ptr()), P(buf.err.data_ptr()), stream,
                                       ctypes.byref(buf.handle_c))
    assert st == moe.OK, moe.moe_status_string(st)
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    eo = bf16_to_dev(np.random.default_rng(5).integers(0, 0x3F80, (buf.rows_cap, H)).astype(np.uint16))
    moe.combine_into(buf.handle_c, eo, y, buf.err)
    assert moe.check() == 0
    out = {n: getattr(buf, n).cpu().numpy() for n in
           ("expert_count", "expert_offset", "rank_offset", "recv_src", "slot")}
    out["recv_x"] = buf.recv_x.view(torch.uint8).cpu().numpy()
    if buf.recv_scale is not None:
        out["recv_scale"] = buf.recv_scale.view(torch.uint8).cpu().numpy()
    out["y"] = bf16_from_dev(y)
    return out, moe.workspace_bytes(cfg, T)


def test_no_alloc_dispatch_matches_moe_dispatch_on_two_calls():
    import combine_route_meta_b200 as moe
    problems = [
        # T, H, E, R, k, fp8, pad128, seed: both large enough for the tiled metadata,
        # which is the part that uses scratch
        (3000, 256, 64, 8, 8, True, True, 1),
        (2600, 512, 256, 32, 8, False, False, 2),
    ]
    for T, H, E, R, k, fp8, pad128, seed in problems:
        x, idx, w = random_problem(seed, T, H, E, k)
        ref, need = _dispatch(moe, "moe_dispatch", x, idx, w, E, R, fp8, pad128)
        got, _ = _dispatch(moe, "moe_dispatch_no_alloc", x, idx, w, E, R, fp8, pad128)
        assert 0 < need <= moe.NO_ALLOC_SCRATCH_BYTES
        for key in ref:
            np.testing.assert_array_equal(got[key], ref[key], err_msg=key)


def test_no_alloc_rejects_problems_beyond_its_scratch():
    import combine_route_meta_b200 as moe
    cfg = moe.make_config(128, 8, 2048, 8, False)
    T = 20000  # 157 tiles x 2048 experts x 4 bytes > 1 MiB
    assert moe.workspace_bytes(cfg, T) > moe.NO_ALLOC_SCRATCH_BYTES
    out = moe.moe_dispatch_out(16, None, 16, 16, 16, 16, T * 8)
    h = moe.moe_handle()
    P = ctypes.c_void_p
    st = moe.moe_dispatch_no_alloc(ctypes.byref(cfg), T, P(16), P(16), P(16), ctypes.byref(out),
                                   P(16), P(16), None, ctypes.byref(h))
    assert st == moe.ERR_TOO_LARGE
    assert b"scratch" in moe.moe_status_string(st)
