"""GPU parity: the CUDA path against the CPU oracle, element by element.

Dispatch (counts, offsets, rank offsets, slots, recv_src, bf16 rows, fp8 codes
and scales) must match bit for bit.  Combine must satisfy, per element,
|y - y_ref| <= 1e-2 + 4e-3 * |y_ref| against the fp64 oracle.  Receive buffers
are filled with a poison byte before the call, on both sides, so rows that
must stay unwritten (padding, unused capacity) are compared too.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests._lib import bf16_from_dev, bf16_to_dev, to_dev
from workloads import (WORKLOADS, bf16_bits_to_f32, f32_to_bf16_bits, make_expert_out,
                       make_inputs, normal_bf16_rows, random_problem)

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 1e-2, 4e-3
POISON = 0xA5

if torch.cuda.is_available():
    import combine_route_meta_b200 as moe


def run_gpu(x, idx, w, *, E, R, fp8, pad128=False, rows_cap=None, inputs_ready=False):
    T, H = x.shape
    k = idx.shape[1]
    cfg = moe.make_config(H, k, E, R, fp8, pad128, inputs_ready)
    buf = moe.Buffers(cfg, T, "cuda", rows_cap)
    buf.recv_x.view(torch.uint8).fill_(POISON)
    if buf.recv_scale is not None:
        buf.recv_scale.view(torch.uint8).fill_(POISON)
    for t in (buf.expert_count, buf.expert_offset, buf.rank_offset, buf.recv_src, buf.slot):
        t.fill_(0x5A5A5A5A)
    moe.check()  # clear the error word
    xd, idd, wd = bf16_to_dev(x), to_dev(idx), to_dev(w)
    moe.dispatch_into(buf, xd, idd, wd)
    bits = moe.check()
    return buf, bits, (xd, idd, wd)


def dispatch_host(buf):
    d = dict(
        expert_count=buf.expert_count.cpu().numpy(),
        expert_offset=buf.expert_offset.cpu().numpy(),
        rank_offset=buf.rank_offset.cpu().numpy(),
        recv_src=buf.recv_src.cpu().numpy(),
        slot=buf.slot.cpu().numpy(),
    )
    if buf.recv_scale is not None:
        d["recv_x"] = buf.recv_x.view(torch.uint8).cpu().numpy()
        d["recv_scale"] = buf.recv_scale.cpu().numpy()
    else:
        d["recv_x"] = bf16_from_dev(buf.recv_x)
    return d


def assert_dispatch_equal(g, o, *, payload=True):
    for key in ("expert_count", "expert_offset", "rank_offset", "slot", "recv_src"):
        np.testing.assert_array_equal(g[key], o[key], err_msg=key)
    if payload:
        np.testing.assert_array_equal(g["recv_x"], o["recv_x"], err_msg="recv_x")
        if "recv_scale" in g:
            np.testing.assert_array_equal(g["recv_scale"].view(np.uint32),
                                          o["recv_scale"].view(np.uint32), err_msg="recv_scale")


def run_combine(buf, expert_out_dev):
    y = torch.empty((buf.T, buf.cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.combine_into(buf.handle_c, expert_out_dev, y, buf.err)
    bits = moe.check()
    return bf16_from_dev(y), bits


def assert_combine_close(y_bits, ref):
    y = bf16_bits_to_f32(y_bits).astype(np.float64)
    err = np.abs(y - ref)
    bound = TOL_ABS + TOL_REL * np.abs(ref)
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{len(bad)} elements out of tolerance, first {bad[:3]}, max err {err.max()}"


def check_problem(x, idx, w, *, E, R, fp8, pad128=False, rows_cap=None, expect_bits=0, inputs_ready=False,
                  expert_out=None):
    buf, bits, _ = run_gpu(x, idx, w, E=E, R=R, fp8=fp8, pad128=pad128, rows_cap=rows_cap,
                           inputs_ready=inputs_ready)
    o = oracle.dispatch(x, idx, E=E, R=R, fp8=fp8, pad128=pad128, rows_cap=buf.rows_cap,
                        recv_fill=POISON)
    assert bits == o["err"] == expect_bits
    g = dispatch_host(buf)
    assert_dispatch_equal(g, o)
    if buf.T == 0:
        return buf, g, o
    if expert_out is None:
        expert_out = normal_bf16_rows(123, 3, 0, buf.rows_cap, x.shape[1])
    y, cbits = run_combine(buf, bf16_to_dev(expert_out))
    assert cbits == 0
    ref = oracle.combine(o["slot"], w, expert_out)
    assert_combine_close(y, ref)
    return buf, g, o


# ---- the named workloads ----------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "dsv3_decode", "kimi_decode", "sweep_256", "sweep_1024",
                                  "prefill_zipf", "sweep_4096"])
def test_workload_parity_full(name):
    w, x, idx, wts = make_inputs(name)
    buf, bits, _ = run_gpu(x, idx, wts, E=w.E, R=w.R, fp8=w.fp8, pad128=w.pad128)
    assert bits == 0
    o = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=w.fp8, pad128=w.pad128, rows_cap=buf.rows_cap,
                        recv_fill=POISON)
    g = dispatch_host(buf)
    assert_dispatch_equal(g, o)
    if w.identity_experts:
        eo_dev, eo_host = buf.recv_x, o["recv_x"]   # each side combines its own dispatched rows
    else:
        eo_host = make_expert_out(w, buf.rows_cap)
        eo_dev = bf16_to_dev(eo_host)
    y, cbits = run_combine(buf, eo_dev)
    assert cbits == 0
    ref = oracle.combine(o["slot"], wts, eo_host)
    assert_combine_close(y, ref)
    if w.identity_experts:
        # y = x * sum_j w_j with sum_j w_j = 1 up to binary32 rounding
        xf = bf16_bits_to_f32(x).astype(np.float64)
        assert np.all(np.abs(bf16_bits_to_f32(y) - xf) <= TOL_ABS + TOL_REL * np.abs(xf))


def test_workload_parity_sampled_largest():
    """T=16384 batch-sweep point: full metadata, sampled payload rows and outputs."""
    w, x, idx, wts = make_inputs("sweep_16384")
    buf, bits, _ = run_gpu(x, idx, wts, E=w.E, R=w.R, fp8=True, pad128=True)
    assert bits == 0
    # metadata does not depend on H: the oracle computes it on a narrow copy of x
    o = oracle.dispatch(x[:, :128], idx, E=w.E, R=w.R, fp8=True, pad128=True, rows_cap=buf.rows_cap)
    g = dispatch_host(buf)
    assert_dispatch_equal(g, o, payload=False)
    rng = np.random.default_rng(77)
    toks = np.unique(np.concatenate([[0, w.T - 1], rng.integers(0, w.T, 61)]))
    for t in toks:
        codes, scales = oracle.quantise_row_fp8(x[t])
        for j in range(w.k):
            s = o["slot"][t, j]
            np.testing.assert_array_equal(g["recv_x"][s], codes)
            np.testing.assert_array_equal(g["recv_scale"][s].view(np.uint32), scales.view(np.uint32))
    # rows that hold no entry stay unwritten (poison)
    pad_rows = np.nonzero(g["recv_src"] == -1)[0]
    sample = pad_rows[rng.integers(0, len(pad_rows), 50)]
    assert np.all(g["recv_x"][sample] == POISON)
    eo_host = make_expert_out(w, buf.rows_cap)
    y, cbits = run_combine(buf, bf16_to_dev(eo_host))
    assert cbits == 0
    ref = oracle.combine(o["slot"], wts, eo_host, tokens=toks)
    assert_combine_close(y[toks], ref)


# ---- shapes and edge cases ----------------------------------------------------------

CASES = [
    # T, H, E, R, k, fp8, pad128, distinct
    # fused one-launch dispatch (S <= 2048, k <= 16): 1, 2 and 4 chunks per warp
    (1, 8, 1, 1, 1, False, False, True),
    (64, 7168, 32, 4, 8, False, True, True),
    (3, 16384, 16, 4, 4, True, False, True),
    (2, 24576, 16, 4, 4, True, True, True),
    (256, 7168, 256, 32, 8, True, True, True),   # S = 2048: the largest fused batch
    # around one resident wave of token CTAs (148 SMs): the launch doubles the
    # chunks per warp when T (+1) CTAs of one chunk would need two waves
    (147, 7168, 256, 8, 8, True, False, True),
    (148, 7168, 256, 8, 8, False, False, True),
    (149, 7168, 256, 8, 8, True, True, True),
    (256, 7168, 256, 8, 8, True, False, True),
    (170, 4096, 128, 8, 12, True, False, False), # k > 8 own ids from shared memory, duplicates
    # past the one-token-per-CTA kernels: the one-launch mid-size kernel for fp8 or
    # narrow bf16 rows with S <= 16384, else metadata kernels + scatter
    (2048, 256, 64, 8, 8, True, True, True),     # S = 16384: the largest mid-size batch
    (2049, 256, 64, 8, 8, True, True, True),     # S = 16392: tiled metadata + fp8 scatter
    (2050, 7680, 64, 8, 8, True, False, True),   # fp8 bulk scatter, 15 chunk warps per row
    (2050, 8192, 64, 8, 8, True, False, True),   # one chunk too many: register scatter
    (700, 1024, 64, 8, 32, True, True, False),   # fp8 bulk scatter, k = 32 slots, duplicates
    (10, 128, 8, 2, 20, False, False, False),
    (600, 1032, 16, 4, 5, False, True, False),   # ragged last 512-column chunk (8 columns)
    (300, 1152, 8, 8, 8, True, True, True),      # 9 scales per row: no 16-byte scale stores
    (3, 30720, 8, 2, 20, True, False, False),    # rows too wide for the bulk stages: register scatter
    (1, 128, 4, 2, 4, True, False, True),
    (5, 136, 6, 3, 3, False, False, True),       # H/8 = 17 vectors: one ragged part
    (33, 1032, 16, 4, 5, False, True, False),    # 129 vectors: two parts, duplicates
    (17, 1152, 8, 8, 2, True, True, True),       # fp8 with 9 blocks per row, R = E
    (700, 384, 64, 8, 8, True, True, True),      # S = 5600: tiled metadata, ragged last tile
    (513, 256, 2048, 16, 8, False, False, True),  # the largest E
    (1000, 128, 32, 4, 64, False, False, False),  # the largest k, duplicates
    (4099, 256, 256, 32, 8, True, True, True),   # S just past 8 tiles
    (2048, 64, 512, 8, 2, False, True, True),    # S = 4096: the largest one-CTA batch
    (2049, 64, 512, 8, 2, False, True, True),    # S = 4098: the smallest tiled batch
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}_H{}_E{}_R{}_k{}_{}{}{}".format(
    *c[:5], "fp8" if c[5] else "bf16", "_pad" if c[6] else "", "" if c[7] else "_dup"))
def test_shapes(case):
    T, H, E, R, k, fp8, pad128, distinct = case
    x, idx, w = random_problem(T * 7 + H, T, H, E, k, distinct=distinct)
    check_problem(x, idx, w, E=E, R=R, fp8=fp8, pad128=pad128)


@pytest.mark.parametrize("fp8,pad128", [(False, False), (True, True)])
def test_empty_batch(fp8, pad128):
    x = np.zeros((0, 256), np.uint16)
    idx = np.zeros((0, 8), np.int32)
    w = np.zeros((0, 8), np.float32)
    buf, g, o = check_problem(x, idx, w, E=16, R=4, fp8=fp8, pad128=pad128, rows_cap=64)
    assert np.all(g["recv_src"] == -1)


@pytest.mark.parametrize("T", [3000, 9000], ids=["mid_size", "tiled"])
def test_every_token_to_one_expert(T):
    # the hot bin: every j = 0 entry on expert 3 and every j = 1 entry on expert 5,
    # which both the mid-size kernel (S = 6000) and the tiled metadata (S = 18000)
    # must still order exactly
    k = 2
    x, _, w = random_problem(41, T, 128, 8, k)
    idx = np.full((T, k), 3, np.int32)
    idx[:, 1] = 5
    check_problem(x, idx, w, E=8, R=2, fp8=False, pad128=True)


def test_every_token_to_one_expert_fused_path():
    # the one-launch kernel's shared-memory counters all hit one expert
    T, k = 200, 2
    x, _, w = random_problem(43, T, 512, 8, k)
    idx = np.full((T, k), 6, np.int32)
    idx[::3, 1] = 1
    check_problem(x, idx, w, E=8, R=4, fp8=True, pad128=True)


def test_zipf_routing_hot_expert_small_H():
    w, x, idx, wts = make_inputs("prefill_zipf", H=256)
    check_problem(x, idx, wts, E=w.E, R=w.R, fp8=True, pad128=False)


@pytest.mark.parametrize("T", [100, 3000])
def test_bad_expert_ids_are_dropped_and_flagged(T):
    x, idx, w = random_problem(5, T, 128, 16, 4)
    idx = idx.copy()
    idx[T // 2, 1] = 16
    idx[T - 1, 3] = -7
    check_problem(x, idx, w, E=16, R=4, fp8=False, expect_bits=moe.DEV_BAD_INDEX)


@pytest.mark.parametrize("T", [50, 2000])
def test_capacity_overflow_is_dropped_and_flagged(T):
    x, idx, w = random_problem(6, T, 128, 8, 4)
    cap = T * 4 - 37
    check_problem(x, idx, w, E=8, R=2, fp8=True, rows_cap=cap, expect_bits=moe.DEV_CAPACITY)


def test_fp8_edge_values():
    # zero blocks, signed zeros, bf16 subnormals, exact e4m3 midpoints after scaling
    T, H = 6, 512
    rng = np.random.default_rng(8)
    xf = (rng.standard_normal((T, H)) * np.exp2(rng.integers(-20, 20, (T, H)))).astype(np.float32)
    xf[0, :128] = 0.0
    xf[1, :128] = -0.0
    xf[1, 128:256] = 0.0
    xf[1, 130] = -0.0
    x = f32_to_bf16_bits(xf)
    x[2, :128] = np.arange(1, 129, dtype=np.uint16)            # positive bf16 subnormals
    x[2, 128:256] = np.arange(1, 129, dtype=np.uint16) | 0x8000  # negative subnormals
    # block with amax 448: scale 1.0, values on midpoints between e4m3 codes
    mids = [0.5 * (a + b) for a, b in [(1.0, 1.125), (1.125, 1.25), (240.0, 256.0), (256.0, 288.0)]]
    blk = np.zeros(128, np.float32)
    blk[0] = 448.0
    blk[1:1 + len(mids)] = mids
    blk[10:20] = -np.array(mids * 3)[:10]
    x[3, :128] = f32_to_bf16_bits(blk)
    idx = np.stack([rng.choice(8, 2, replace=False) for _ in range(T)]).astype(np.int32)
    w = np.full((T, 2), 0.5, np.float32)
    check_problem(x, idx, w, E=8, R=2, fp8=True)


def test_one_hot_weights_combine_is_exact():
    x, idx, _ = random_problem(9, 300, 256, 16, 4)
    buf, _, _ = run_gpu(x, idx, np.zeros((300, 4), np.float32), E=16, R=4, fp8=False)
    eo = make_expert_out(WORKLOADS["tiny"], buf.rows_cap)
    for j in range(4):
        w = np.zeros((300, 4), np.float32)
        w[:, j] = 1.0
        buf2, _, _ = run_gpu(x, idx, w, E=16, R=4, fp8=False)
        y, _ = run_combine(buf2, bf16_to_dev(eo))
        np.testing.assert_array_equal(bf16_bits_to_f32(y), bf16_bits_to_f32(eo[buf2.slot.cpu().numpy()[:, j]]))


def test_runs_are_bitwise_deterministic():
    w, x, idx, wts = make_inputs("prefill_zipf", H=1024)
    outs = []
    for _ in range(2):
        buf, bits, _ = run_gpu(x, idx, wts, E=w.E, R=w.R, fp8=True, pad128=True)
        g = dispatch_host(buf)
        eo = bf16_to_dev(make_expert_out(w, buf.rows_cap))
        y, _ = run_combine(buf, eo)
        outs.append((g, y))
    for key in outs[0][0]:
        np.testing.assert_array_equal(outs[0][0][key], outs[1][0][key])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("name,over", [("dsv3_decode", {}), ("sweep_1024", {}),
                                       ("sweep_4096", {"H": 512})],
                         ids=["one_token_per_cta", "mid_size", "tiled"])
def test_graph_capture_replays_the_same_result(name, over):
    # no host read-back inside dispatch/combine: the pair can be captured and replayed
    w, x, idx, wts = make_inputs(name, **over)
    cfg = moe.make_config(w.H, w.k, w.E, w.R, w.fp8, w.pad128)
    buf = moe.Buffers(cfg, w.T, "cuda")
    xd, idd, wd = bf16_to_dev(x), to_dev(idx), to_dev(wts)
    eo = bf16_to_dev(make_expert_out(w, buf.rows_cap))
    y = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.dispatch_into(buf, xd, idd, wd, stream=s)   # warm-up outside capture
        moe.combine_into(buf.handle_c, eo, y, buf.err, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.dispatch_into(buf, xd, idd, wd)
        moe.combine_into(buf.handle_c, eo, y, buf.err)
    buf.recv_x.view(torch.uint8).fill_(0)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    o = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=w.fp8, pad128=w.pad128, rows_cap=buf.rows_cap)
    gd = dispatch_host(buf)
    np.testing.assert_array_equal(gd["slot"], o["slot"])
    valid = o["recv_src"] >= 0
    np.testing.assert_array_equal(gd["recv_x"][valid], o["recv_x"][valid])
    ref = oracle.combine(o["slot"], wts, bf16_from_dev(eo))
    assert_combine_close(bf16_from_dev(y), ref)
    assert moe.check() == 0


def test_graph_capture_of_router_then_dispatch():
    # router + dispatch in one call, captured: the replay routes and dispatches afresh
    T, E, R, k, H = 128, 256, 8, 8, 7168
    rng = np.random.default_rng(17)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    cfg = moe.make_config(H, k, E, R, True, False)
    buf = moe.Buffers(cfg, T, "cuda")
    ld, xd = to_dev(logits), bf16_to_dev(x)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.route_dispatch_into(buf, xd, ld, idx, wt, score_fn="sigmoid", n_group=8, topk_group=4,
                                stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.route_dispatch_into(buf, xd, ld, idx, wt, score_fn="sigmoid", n_group=8, topk_group=4)
    idx.fill_(-1)
    buf.slot.fill_(-5)
    g.replay()
    torch.cuda.synchronize()
    ref_idx, _ = oracle.router_topk(logits, k, score_fn="sigmoid", n_group=8, topk_group=4)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    o = oracle.dispatch(x, ref_idx, E=E, R=R, fp8=True, rows_cap=buf.rows_cap)
    np.testing.assert_array_equal(buf.slot.cpu().numpy(), o["slot"])
    assert moe.check() == 0


def test_torch_level_api():
    w, x, idx, wts = make_inputs("tiny")
    xd = bf16_to_dev(x)
    d = moe.dispatch(xd, to_dev(idx).long(), to_dev(wts), num_experts=w.E,
                     num_virtual_ranks=w.R, fp8=False)
    y = moe.combine(d.handle, d.recv_x)
    assert moe.check() == 0
    o = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=False)
    np.testing.assert_array_equal(d.expert_offset.cpu().numpy(), o["expert_offset"])
    assert_combine_close(bf16_from_dev(y), oracle.combine(o["slot"], wts, o["recv_x"]))


def _all_bf16_blocks(rng):
    """Rows of 128-column blocks: each block starts with its amax A and then walks through
    every bf16 value of magnitude <= A (both signs), for about 30 amax values A."""
    amaxes = [0x0040, 0x0080, 0x0101, 0x1F35, 0x2F00, 0x3A8F, 0x3B80, 0x3C00, 0x3D4D, 0x3E80,
              0x3F00, 0x3F80, 0x3FC9, 0x4000, 0x4049, 0x40A0, 0x4120, 0x41A0, 0x4300, 0x43E0,
              0x4400, 0x4500, 0x4680, 0x4780, 0x4B00, 0x5000, 0x5A5A, 0x6000, 0x7000, 0x7F7F]
    blocks = []
    for a in amaxes:
        vals = np.arange(0, a + 1, dtype=np.uint32)
        vals = np.concatenate([vals, vals | 0x8000]).astype(np.uint16)
        rng.shuffle(vals)
        n = (len(vals) + 126) // 127
        vals = np.resize(vals, n * 127)
        blk = np.empty((n, 128), np.uint16)
        blk[:, 0] = a if rng.random() < 0.5 else a | 0x8000
        blk[:, 1:] = vals.reshape(n, 127)
        blocks.append(blk)
    blocks = np.concatenate(blocks)
    per_row = 64
    rows = (len(blocks) + per_row - 1) // per_row
    blocks = np.resize(blocks, (rows * per_row, 128))
    return blocks.reshape(rows, per_row * 128)


@pytest.mark.parametrize("k", [1, 17], ids=["fused", "scatter"])
def test_fp8_quantiser_every_bf16_value(k):
    # every bf16 magnitude below each block's amax, through the kernel's quotient shortcut and
    # its exact fallback; codes and scales must equal the oracle's bit for bit
    rng = np.random.default_rng(2024)
    x = _all_bf16_blocks(rng)
    T = x.shape[0]
    idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    w = np.full((T, k), 1.0 / k, np.float32)
    buf, bits, _ = run_gpu(x, idx, w, E=k, R=1, fp8=True)
    assert bits == 0
    g = dispatch_host(buf)
    for t in range(T):
        codes, scales = oracle.quantise_row_fp8(x[t])
        for j in (0, k - 1):
            s = g["slot"][t, j]
            np.testing.assert_array_equal(g["recv_x"][s], codes, err_msg=f"row {t}")
            np.testing.assert_array_equal(g["recv_scale"][s].view(np.uint32), scales.view(np.uint32))


def test_bounded_wait_reports_timeout_and_context_survives():
    # a wait on a barrier nothing completes gives up after its limit and reports the bit
    err = moe.error_word()
    moe.check()
    st = moe.moe_selftest_bounded_wait(ctypes.c_void_p(err.data_ptr()), 20_000_000,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.OK
    assert moe.check() == moe.DEV_TIMEOUT
    # the context is still usable: a normal dispatch + combine matches the oracle
    x, idx, w = random_problem(12, 64, 512, 8, 2)
    check_problem(x, idx, w, E=8, R=2, fp8=True)


@pytest.mark.parametrize("T,H,E,k,fp8,pad128", [(40, 256, 8, 4, True, False),       # one-CTA layout
                                                (3000, 1024, 64, 8, False, True),   # tiled, bulk bf16
                                                (700, 7168, 256, 8, True, True)])   # tiled, fp8
def test_layout_then_payload_equals_dispatch(T, H, E, k, fp8, pad128):
    x, idx, w = random_problem(T + H, T, H, E, k)
    ref, bits, _ = run_gpu(x, idx, w, E=E, R=E // 4 or 1, fp8=fp8, pad128=pad128)
    assert bits == 0
    cfg = moe.make_config(H, k, E, E // 4 or 1, fp8, pad128)
    buf = moe.Buffers(cfg, T, "cuda")
    buf.recv_x.view(torch.uint8).fill_(POISON)
    if buf.recv_scale is not None:
        buf.recv_scale.view(torch.uint8).fill_(POISON)
    idd, xd = to_dev(idx), bf16_to_dev(x)
    moe.dispatch_layout_into(buf, idd)
    moe.dispatch_payload_into(buf, xd)
    assert moe.check() == 0
    a, b = dispatch_host(buf), dispatch_host(ref)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)


@pytest.mark.parametrize("T,H,E,R,k,fp8,pad128", [
    (300, 1152, 8, 8, 8, True, True),      # S = 2400: one-CTA layout
    (2048, 64, 512, 8, 2, False, True),    # S = 4096: the largest one-CTA layout
    (2049, 64, 512, 8, 2, False, True),    # S = 4098: the smallest tiled layout
    (5000, 128, 256, 32, 8, True, False),  # tiled, several tiles
])
def test_layout_path_matches_oracle(T, H, E, R, k, fp8, pad128):
    # moe_dispatch takes the one-launch kernel at these sizes; the separate
    # layout and payload calls keep the one-CTA and tiled metadata kernels, which
    # are compared with the oracle here
    x, idx, w = random_problem(T * 3 + H, T, H, E, k, distinct=E >= k)
    if T == 5000:
        idx[: T // 2, 0] = 7  # a hot expert across many tiles
    cfg = moe.make_config(H, k, E, R, fp8, pad128)
    buf = moe.Buffers(cfg, T, "cuda")
    buf.recv_x.view(torch.uint8).fill_(POISON)
    if buf.recv_scale is not None:
        buf.recv_scale.view(torch.uint8).fill_(POISON)
    moe.check()
    moe.dispatch_layout_into(buf, to_dev(idx))
    moe.dispatch_payload_into(buf, bf16_to_dev(x))
    assert moe.check() == 0
    o = oracle.dispatch(x, idx, E=E, R=R, fp8=fp8, pad128=pad128, rows_cap=buf.rows_cap,
                        recv_fill=POISON)
    assert_dispatch_equal(dispatch_host(buf), o)


@pytest.mark.parametrize("H,fp8", [(256, False), (2048, False), (512, True)])
def test_payload_skips_and_flags_bad_slots(H, fp8):
    # register scatter (H=256), bulk scatter (bf16, H=2048) and fp8: slots outside
    # [-1, rows_cap) are skipped and flagged; nothing outside the buffers is touched
    T, k = 20, 2
    x, _, _ = random_problem(3, T, H, 8, k)
    cfg = moe.make_config(H, k, 8, 2, fp8)
    buf = moe.Buffers(cfg, T, "cuda", rows_cap=T * k)
    buf.recv_x.view(torch.uint8).fill_(POISON)
    slot = np.arange(T * k, dtype=np.int32).reshape(T, k)
    slot[3, 1] = T * k          # one past the end
    slot[5, 0] = -7             # negative, not -1
    slot[6, 1] = -1             # "no row": skipped silently
    moe.check()
    moe.dispatch_payload_into(buf, bf16_to_dev(x), to_dev(slot))
    assert moe.check() == moe.DEV_BAD_SLOT
    got = buf.recv_x.view(torch.uint8).cpu().numpy().reshape(T * k, -1)
    # each row r was meant for entry r; the three entries without a valid slot left theirs alone
    for r in (3 * k + 1, 5 * k + 0, 6 * k + 1):
        assert np.all(got[r] == POISON), r
    if not fp8:
        for t in (0, 7, T - 1):
            for j in range(k):
                np.testing.assert_array_equal(got[slot[t, j]].view(np.uint16), x[t])


@pytest.mark.parametrize("T,H,E,R,k,fp8,pad128", [
    (300, 7168, 64, 8, 8, True, False),      # fp8 bulk row stores
    (257, 512, 32, 4, 6, True, True),        # one chunk warp per row, padding
    (90, 1152, 16, 4, 4, True, False),       # 9 scales per row: register scatter
    (300, 2048, 64, 8, 8, False, False),     # bf16 bulk scatter
])
def test_layout_then_payload_equals_the_oracle(T, H, E, R, k, fp8, pad128):
    # the two phases as separate calls (the payload kernels that do not load x
    # before the previous kernel finishes)
    x, idx, w = random_problem(T * H, T, H, E, k)
    cfg = moe.make_config(H, k, E, R, fp8, pad128)
    buf = moe.Buffers(cfg, T, "cuda")
    buf.recv_x.view(torch.uint8).fill_(POISON)
    if buf.recv_scale is not None:
        buf.recv_scale.view(torch.uint8).fill_(POISON)
    moe.check()
    moe.dispatch_layout_into(buf, to_dev(idx))
    moe.dispatch_payload_into(buf, bf16_to_dev(x))
    assert moe.check() == 0
    o = oracle.dispatch(x, idx, E=E, R=R, fp8=fp8, pad128=pad128, rows_cap=buf.rows_cap, recv_fill=POISON)
    assert_dispatch_equal(dispatch_host(buf), o)


@pytest.mark.parametrize("T,H,E,R,k,fp8,distinct,bad,cap", [
    (128, 7168, 256, 8, 8, True, True, False, None),     # DeepSeek-V3-shaped decode
    (128, 7168, 384, 16, 8, True, True, False, None),    # Kimi-K2-shaped decode
    (64, 4096, 128, 8, 12, True, False, False, None),    # 16 own ids, duplicates
    (100, 2048, 64, 4, 8, False, True, False, None),     # bf16 rows
    (40, 1024, 32, 4, 4, True, True, True, None),        # bad ids: flagged after the wait
    (50, 1024, 16, 4, 4, False, True, False, 120),       # capacity short of T*k
])
def test_inputs_ready_dispatch(T, H, E, R, k, fp8, distinct, bad, cap):
    # MOE_INPUTS_READY: the decode kernel reads and computes before waiting for
    # the previous kernel and writes after; the results are those of moe_dispatch
    x, idx, w = random_problem(T + k, T, H, E, k, distinct=distinct)
    if bad:
        idx[3, 1] = E + 2
        idx[T - 1, 0] = -1
    bits = (moe.DEV_BAD_INDEX if bad else 0) | (moe.DEV_CAPACITY if cap is not None else 0)
    check_problem(x, idx, w, E=E, R=R, fp8=fp8, rows_cap=cap, expect_bits=bits, inputs_ready=True)
