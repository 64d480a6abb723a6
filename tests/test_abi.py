"""The C ABI without a GPU: the library loads, exports what the header declares,
and its host-only calls (sizing, argument validation) behave as documented."""
import ctypes
import re

import pytest

import oracle
from tests._lib import HEADER

import combine_route_meta_b200 as moe


def _declared():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(_declared())
    for n in ["moe_dispatch", "moe_combine", "moe_rows_capacity", "moe_workspace_bytes",
              "moe_dispatch_sizes_for", "moe_check", "moe_status_string", "moe_version"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(moe.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_mirrors_c_names():
    for name in _declared():
        assert callable(getattr(moe, name)), name


def test_version_and_status_strings():
    assert moe.moe_version() >= 100
    assert moe.moe_status_string(moe.OK) == b"ok"
    assert moe.moe_status_string(moe.ERR_UNSUPPORTED) == b"unsupported configuration"


@pytest.mark.parametrize("T,k,E,pad", [(0, 8, 256, True), (1, 1, 4, True), (16, 2, 8, False),
                                       (128, 8, 256, False), (256, 8, 256, True),
                                       (1024, 8, 256, True), (16384, 8, 256, True),
                                       (3, 2, 1, True), (7, 3, 1000, True)])
def test_rows_capacity_matches_oracle(T, k, E, pad):
    cfg = moe.make_config(128, k, E, 1, fp8=False, pad128=pad)
    assert moe.rows_capacity(cfg, T) == oracle.rows_capacity(T, k, E, pad)


def test_config_validation_statuses():
    bad = [
        (moe.make_config(0, 8, 256, 8, False), moe.ERR_INVALID_ARG),
        (moe.make_config(7168, 0, 256, 8, False), moe.ERR_INVALID_ARG),
        (moe.make_config(7168, 8, 256, 7, False), moe.ERR_INVALID_ARG),   # E % R
        (moe.make_config(7168, 8, 0, 1, False), moe.ERR_INVALID_ARG),
        (moe.make_config(100, 8, 256, 8, False), moe.ERR_UNSUPPORTED),    # H % 8
        (moe.make_config(7176, 8, 256, 8, True), moe.ERR_UNSUPPORTED),    # fp8 needs H % 128
        (moe.make_config(128, 8, 4096, 8, False), moe.ERR_UNSUPPORTED),   # E > max
        (moe.make_config(128, 65, 256, 8, False), moe.ERR_UNSUPPORTED),   # k > max
    ]
    for cfg, want in bad:
        sizes = moe.moe_dispatch_sizes()
        assert moe.moe_dispatch_sizes_for(ctypes.byref(cfg), 4, 32, ctypes.byref(sizes)) == want
        assert moe.moe_rows_capacity(ctypes.byref(cfg), 4) == -1
    for bit in (8, 1 << 30):  # flag bits the header does not define
        cfg = moe.moe_config(128, 2, 8, 2, bit)
        assert moe.moe_rows_capacity(ctypes.byref(cfg), 4) == -1
    cfg = moe.moe_config(128, 2, 8, 2, moe.INPUTS_READY)
    assert moe.moe_rows_capacity(ctypes.byref(cfg), 4) > 0


def test_dispatch_rejects_bad_arguments_before_touching_the_gpu():
    cfg = moe.make_config(256, 2, 8, 2, fp8=False)
    out = moe.moe_dispatch_out(16, None, 16, 16, 16, 16, 32)
    h = moe.moe_handle()
    P = ctypes.c_void_p
    # null error word
    assert moe.moe_dispatch(ctypes.byref(cfg), 16, P(16), P(16), P(16), ctypes.byref(out), P(16),
                            None, 0, None, None, ctypes.byref(h)) == moe.ERR_INVALID_ARG
    # misaligned x
    assert moe.moe_dispatch(ctypes.byref(cfg), 16, P(18), P(16), P(16), ctypes.byref(out), P(16),
                            None, 0, P(16), None, ctypes.byref(h)) == moe.ERR_INVALID_ARG
    # negative T
    assert moe.moe_dispatch(ctypes.byref(cfg), -1, P(16), P(16), P(16), ctypes.byref(out), P(16),
                            None, 0, P(16), None, ctypes.byref(h)) == moe.ERR_INVALID_ARG
    # missing workspace for a batch that needs one
    big = moe.make_config(256, 8, 8, 2, fp8=False)
    assert moe.workspace_bytes(big, 4096) > 0
    out2 = moe.moe_dispatch_out(16, None, 16, 16, 16, 16, 4096 * 8)
    assert moe.moe_dispatch(ctypes.byref(big), 4096, P(16), P(16), P(16), ctypes.byref(out2), P(16),
                            None, 0, P(16), None, ctypes.byref(h)) == moe.ERR_INVALID_ARG
    # fp8 without a scale buffer
    f8 = moe.make_config(256, 2, 8, 2, fp8=True)
    assert moe.moe_dispatch(ctypes.byref(f8), 16, P(16), P(16), P(16), ctypes.byref(out), P(16),
                            None, 0, P(16), None, ctypes.byref(h)) == moe.ERR_INVALID_ARG


def test_route_dispatch_checks_both_steps_before_launching():
    # every case fails a check of the router or of the dispatch, so nothing runs
    cfg = moe.make_config(256, 2, 8, 2, fp8=False)
    out = moe.moe_dispatch_out(16, None, 16, 16, 16, 16, 32)
    h = moe.moe_handle()
    P = ctypes.c_void_p
    def call(c=cfg, T=16, logits=P(16), fn=moe.SCORE_SOFTMAX, G=1, TG=1, err=P(16), x=P(16)):
        return moe.moe_route_dispatch(ctypes.byref(c), T, x, logits, fn, G, TG, 1, P(16), P(16),
                                      ctypes.byref(out), P(16), None, 0, err, None, ctypes.byref(h))
    assert call(logits=None) == moe.ERR_INVALID_ARG          # router: no logits
    assert call(fn=7) == moe.ERR_INVALID_ARG                  # router: unknown score function
    assert call(G=3) == moe.ERR_INVALID_ARG                   # router: groups do not divide E
    assert call(G=8, TG=1) == moe.ERR_INVALID_ARG             # router: k > topk_group * E / n_group
    assert call(err=None) == moe.ERR_INVALID_ARG              # dispatch: no error word
    assert call(x=P(18)) == moe.ERR_INVALID_ARG               # dispatch: misaligned x
    assert call(T=-1) == moe.ERR_INVALID_ARG
    wide = moe.make_config(256, 2, 2048, 2, fp8=False)        # E beyond the router's limit
    assert call(c=wide) == moe.ERR_UNSUPPORTED


def test_expert_parallel_calls_check_their_arguments():
    P = ctypes.c_void_p
    cfg = moe.make_config(256, 2, 16, 4, fp8=False)                 # W = 4 ranks
    assert moe.ep_rows_capacity(cfg, 10) == 4 * 10 * 2
    pad = moe.make_config(256, 2, 16, 4, fp8=False, pad128=True)
    assert moe.ep_rows_capacity(pad, 10) == (80 + 127 * 4) // 128 * 128   # 4 local experts
    many = moe.make_config(256, 2, 128, 128, fp8=False)              # more ranks than supported
    assert moe.moe_ep_rows_capacity(ctypes.byref(many), 10) == -1
    args = [P(16)] * 4
    # rank outside [0, W)
    assert moe.moe_ep_layout(ctypes.byref(cfg), 4, 10, *args, 100, P(16), P(16), P(16), P(16),
                             None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_layout(ctypes.byref(many), 0, 10, *args, 100, P(16), P(16), P(16), P(16),
                             None) == moe.ERR_UNSUPPORTED
    table = (P * 4)(16, 32, None, 48)                                 # a missing peer buffer
    assert moe.moe_ep_dispatch_payload(ctypes.byref(cfg), 10, P(16), P(16), P(16), table, None, 100,
                                       0, None, None, None, P(16), None) == moe.ERR_INVALID_ARG
    table = (P * 4)(16, 32, 40, 48)                                   # a misaligned one
    assert moe.moe_ep_dispatch_payload(ctypes.byref(cfg), 10, P(16), P(16), P(16), table, None, 100,
                                       0, None, None, None, P(16), None) == moe.ERR_INVALID_ARG
    f8 = moe.make_config(256, 2, 16, 4, fp8=True)                     # fp8 without scale buffers
    table = (P * 4)(16, 32, 64, 48)
    assert moe.moe_ep_dispatch_payload(ctypes.byref(f8), 10, P(16), P(16), P(16), table, None, 100,
                                       0, None, None, None, P(16), None) == moe.ERR_INVALID_ARG
    flags = (P * 4)(16, 32, 64, 48)
    # signalling: rank outside [0, W), missing epoch or done count, a missing peer flag array
    for rank, ep, done, fl in [(4, P(16), P(16), flags), (0, None, P(16), flags), (0, P(16), None, flags),
                               (0, P(16), P(16), (P * 4)(16, None, 64, 48))]:
        assert moe.moe_ep_dispatch_payload(ctypes.byref(cfg), 0, None, None, None, None, None, 100,
                                           rank, fl, ep, done, P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_signal(0, 0, flags, P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_signal(4, 4, flags, P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_signal(4, 0, (P * 4)(16, 32, None, 48), P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_signal(4, 0, flags, None, None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_wait(4, P(16), P(16), 0, P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_wait(4, P(16), P(16), 10_000_000_001, P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_wait(65, P(16), P(16), 1000, P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_wait(4, None, P(16), 1000, P(16), None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_wait(4, P(16), P(16), 1000, None, None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_combine(ctypes.byref(cfg), 10, P(16), P(16), P(16), None, 100, P(16), P(16),
                              None) == moe.ERR_INVALID_ARG
    assert moe.moe_ep_combine(ctypes.byref(cfg), 10, P(16), P(16), P(16), table, -1, P(16), P(16),
                              None) == moe.ERR_INVALID_ARG


def test_combine_rejects_bad_arguments():
    h = moe.moe_handle(moe.make_config(256, 2, 8, 2, False), 16, 16, 16, 32)
    P = ctypes.c_void_p
    assert moe.moe_combine(None, P(16), P(16), None, None) == moe.ERR_INVALID_ARG
    assert moe.moe_combine(ctypes.byref(h), P(16), None, None, None) == moe.ERR_INVALID_ARG
    assert moe.moe_combine(ctypes.byref(h), P(8), P(16), None, None) == moe.ERR_INVALID_ARG
    h.T = 0  # nothing to do: returns without launching
    assert moe.moe_combine(ctypes.byref(h), None, None, None, None) == moe.OK


def test_sizes_for_fp8():
    cfg = moe.make_config(7168, 8, 256, 8, fp8=True)
    s = moe.moe_dispatch_sizes()
    assert moe.moe_dispatch_sizes_for(ctypes.byref(cfg), 128, 1024, ctypes.byref(s)) == moe.OK
    assert s.recv_x == 1024 * 7168 and s.recv_scale == 1024 * 56 * 4
    assert s.expert_offset == 257 * 4 and s.rank_offset == 9 * 4 and s.slot == 128 * 8 * 4


def test_selftest_wait_rejects_bad_limits():
    P = ctypes.c_void_p
    assert moe.moe_selftest_bounded_wait(None, 1000, None) == moe.ERR_INVALID_ARG
    assert moe.moe_selftest_bounded_wait(P(16), 0, None) == moe.ERR_INVALID_ARG
    assert moe.moe_selftest_bounded_wait(P(16), 2_000_000_000, None) == moe.ERR_INVALID_ARG


@pytest.mark.parametrize("W,E,k,T", [(2, 4, 2, 3), (4, 8, 3, 2), (2, 2, 1, 5), (3, 9, 2, 2)])
def test_ep_rows_capacity_is_the_worst_case(W, E, k, T):
    # every way W ranks' entries (T tokens, k each) can land on one rank's E/W
    # experts: the padded capacity is the most 128-row blocks they can fill,
    # reached by spreading single entries over as many experts as possible
    import itertools
    import math
    El = E // W
    S = W * T * k
    worst = 0
    for n_experts in range(1, min(El, S) + 1):
        # split S entries over n_experts non-empty experts; padding rounds each up
        for parts in itertools.combinations_with_replacement(range(1, S + 1), n_experts):
            if sum(parts) != S:
                continue
            worst = max(worst, sum(math.ceil(p / 128) * 128 for p in parts))
    pad = moe.make_config(256, k, E, W, fp8=False, pad128=True)
    assert moe.ep_rows_capacity(pad, T) == worst
    plain = moe.make_config(256, k, E, W, fp8=False)
    assert moe.ep_rows_capacity(plain, T) == S
