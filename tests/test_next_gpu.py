"""GPU parity of the rows next to dispatch/combine: sender-side partial combine,
expert-side SiLU + block-fp8 quantiser, and the router top-k.  Each is compared
with the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from tests._lib import bf16_from_dev, bf16_to_dev, silu_pairs_near_rounding_boundaries, to_dev
from workloads import (WORKLOADS, bf16_bits_to_f32, f32_to_bf16_bits, make_inputs,
                       make_router_logits, normal_bf16_rows, random_problem)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import combine_route_meta_b200 as moe


def _bf16_ulp(v):
    a = np.abs(v.astype(np.float64))
    return np.where(a == 0, 2.0 ** -133, np.exp2(np.floor(np.log2(np.maximum(a, 1e-300))) - 7))


# ---- sender-side (per-rank) partial combine -------------------------------------

@pytest.mark.parametrize("name,E,R,H,T,k", [("dsv3_decode", 256, 8, 7168, None, 8),
                                            ("kimi_decode", 384, 16, 7168, None, 8),
                                            ("random", 16, 16, 1032, 300, 8),
                                            ("random", 64, 1, 256, 500, 8),
                                            ("random", 64, 4, 2048, 3000, 8),
                                            ("random", 64, 8, 512, 200, 12),   # rows loaded per partial
                                            ("random", 128, 16, 256, 100, 40)])  # layout by one thread
def test_rank_partial_combine(name, E, R, H, T, k):
    if name == "random":
        x, idx, w = random_problem(E + T, T, H, E, k)
        fp8 = False
    else:
        wl, x, idx, w = make_inputs(name)
        fp8 = wl.fp8
    d = moe.dispatch(bf16_to_dev(x), to_dev(idx), to_dev(w), E, R, fp8)
    rows = d.recv_x.shape[0]
    eo = normal_bf16_rows(7, 3, 0, rows, H)
    y, partial, prank, npart = moe.combine_rank_partial(d.handle, d.rank_offset, bf16_to_dev(eo))
    assert moe.check() == 0
    slot = d.handle.slot.cpu().numpy()
    o = oracle.combine_rank_partial(idx, slot, w, eo, E=E, R=R)
    np.testing.assert_array_equal(npart.cpu().numpy(), o["npart"])
    gp = bf16_from_dev(partial)
    n = o["npart"]
    # magnitude of the terms summed into token t's partials: sum_j |w_j| |row_j|
    kept = slot >= 0
    rows_abs = np.abs(bf16_bits_to_f32(eo).astype(np.float64))
    mag = np.zeros((idx.shape[0], H))
    for j in range(idx.shape[1]):
        m = kept[:, j]
        mag[m] += np.abs(w[m, j].astype(np.float64))[:, None] * rows_abs[slot[m, j]]
    # a binary32 chain of at most k fused multiply-adds is within k 2^-24 mag of the
    # exact sum; rounding both to bf16 adds one unit of the larger result
    k_eff = idx.shape[1]
    for t in range(idx.shape[0]):
        np.testing.assert_array_equal(prank.cpu().numpy()[t, :n[t]], o["partial_rank"][t, :n[t]])
        a = bf16_bits_to_f32(gp[t, :n[t]]).astype(np.float64)
        b = bf16_bits_to_f32(o["partial"][t, :n[t]]).astype(np.float64)
        tol = np.maximum(_bf16_ulp(a), _bf16_ulp(b)) + 2.0 * k_eff * 2.0 ** -24 * mag[t]
        assert np.all(np.abs(a - b) <= tol), t
    # stage 2: y is the bf16 rounding of the GPU's own partials summed in binary32, q ascending
    acc = np.zeros((idx.shape[0], H), np.float32)
    for q in range(idx.shape[1]):
        m = q < n
        acc[m] += bf16_bits_to_f32(gp[m, q])
    want = torch.from_numpy(acc).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bf16_from_dev(y), want)
    # and against the oracle's y: the combine tolerance plus the partials' rounding
    yf = bf16_bits_to_f32(bf16_from_dev(y)).astype(np.float64)
    slack = np.abs(bf16_bits_to_f32(o["partial"]).astype(np.float64))
    bound = 1e-2 + 4e-3 * np.abs(o["y"]) + (_bf16_ulp(bf16_bits_to_f32(o["partial"])) * (slack > 0)).sum(1)
    assert np.all(np.abs(yf - o["y"]) <= bound)


# ---- expert-side SiLU + block-fp8 quantiser ---------------------------------------

def _silu_problem(rows, I, seed, pad_frac=0.2):
    rng = np.random.default_rng(seed)
    gu = f32_to_bf16_bits((rng.standard_normal((rows, 2 * I)) * 2).astype(np.float32))
    src = np.arange(rows, dtype=np.int32)
    src[rng.random(rows) < pad_frac] = -1
    return gu, src


@pytest.mark.parametrize("rows,I,in_use,col_major", [(1024, 2048, 1000, False), (1024, 2048, 1024, True),
                                                     (300, 384, 299, False), (70, 1152, 0, False),
                                                     (4096, 2048, 4000, True), (8192, 1024, 8000, False)])
def test_silu_quant_bit_exact(rows, I, in_use, col_major):
    gu, src = _silu_problem(rows, I, rows + I)
    act_ref, sc_ref = oracle.silu_quant(gu, src, in_use, col_major=col_major, fill=0xA5)
    shape = (I // 128, rows) if col_major else (rows, I // 128)
    act = torch.full((rows, I), 0xA5, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(shape, dtype=torch.float32, device="cuda")
    sc.view(torch.uint8).fill_(0xA5)
    moe.silu_quant_into(bf16_to_dev(gu), to_dev(src), to_dev(np.array([in_use], np.int32)),
                        act, sc, col_major=col_major)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(act.cpu().numpy(), act_ref)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), sc_ref.view(np.uint32))


def test_silu_quant_every_bf16_gate_value():
    # gate runs through every finite bf16 value (up = 1), so the activation is
    # checked against the oracle's on its whole input domain
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    I = 2048
    rows = (len(bits) + I - 1) // I
    g = np.resize(bits, rows * I).reshape(rows, I)
    gu = np.concatenate([g, np.full((rows, I), 0x3F80, np.uint16)], axis=1)
    src = np.arange(rows, dtype=np.int32)
    act_ref, sc_ref = oracle.silu_quant(gu, src, rows)
    act, sc = moe.silu_quant(bf16_to_dev(gu), to_dev(src), to_dev(np.array([rows], np.int32)))
    np.testing.assert_array_equal(act.view(torch.uint8).cpu().numpy(), act_ref)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), sc_ref.view(np.uint32))


def _finite_bf16_bits():
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    return bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)


def _silu_mul_dev(gb, ub, **kw):
    return moe.silu_mul(bf16_to_dev(gb), bf16_to_dev(ub), **kw)


@pytest.mark.parametrize("exact_only", [False, True])
def test_silu_activation_every_bf16_gate_value(exact_only):
    # both tiers of the kernel (certified fp64, and double-double alone) give the
    # correctly rounded activation on every finite bf16 gate, for up values from
    # tiny to large
    bits = _finite_bf16_bits()
    for ub in (0x3F80, 0xC0A3, 0x0001, 0x0B17, 0x5F3A, 0xF1C4, 0x8000):
        u = np.full(bits.shape, ub, np.uint16)
        got = _silu_mul_dev(bits, u, exact_only=exact_only).cpu().numpy()
        want = oracle.silu_mul_bits(bits, u)
        bad = np.nonzero(got.view(np.uint32) != want.view(np.uint32))[0]
        assert bad.size == 0, (hex(ub), [(float(bf16_bits_to_f32(bits[i])), got[i], want[i]) for i in bad[:5]])


def test_silu_activation_next_to_rounding_boundaries():
    # pairs within 2^-36 of a binary32 halfway point: many fall inside the fast
    # tier's margin, so the double-double tier decides them
    gb, ub = silu_pairs_near_rounding_boundaries()
    for shift in (0, 40, -60, -120):
        us = (ub.astype(np.int32) + (shift << 7)).astype(np.uint16)
        got, fast = _silu_mul_dev(gb, us, with_fast_value=True)
        got, fast = got.cpu().numpy(), fast.cpu().numpy()
        want = oracle.silu_mul_bits(gb, us)
        np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
        low = (fast.view(np.uint64) & np.uint64((1 << 29) - 1)).astype(np.int64)
        uncertified = np.abs(low - (1 << 28)) <= 32
        if shift == 0:
            assert uncertified.sum() > 50          # the exact tier is exercised


def test_silu_fast_tier_error_bound():
    # the fast tier's fp64 value is within 1.5 * 2^-50 (relative) of the real
    # g u / (1 + e^-g): checked against 50-digit decimal arithmetic on every bf16
    # gate in [-200, 200] with u = 1, and on pairs next to rounding boundaries
    from decimal import Context, Decimal
    ctx = Context(prec=50, Emax=10**6, Emin=-10**6)
    bits = _finite_bf16_bits()
    g = bf16_bits_to_f32(bits).astype(np.float64)
    sel = (g >= -200) & (g <= 200) & (np.abs(g) >= 2.0 ** -126)
    gb, ub = silu_pairs_near_rounding_boundaries()
    gb = np.concatenate([bits[sel], gb])
    ub = np.concatenate([np.full(int(sel.sum()), 0x3F80, np.uint16), ub])
    _, fast = _silu_mul_dev(gb, ub, with_fast_value=True)
    fast = fast.cpu().numpy()
    gv, uv = bf16_bits_to_f32(gb), bf16_bits_to_f32(ub)
    worst = 0.0
    for i in range(len(gb)):
        G, U = Decimal(float(gv[i])), Decimal(float(uv[i]))
        exact = ctx.divide(ctx.multiply(G, U), ctx.add(1, ctx.exp(-G)))
        rel = abs((Decimal(float(fast[i])) - exact) / exact)
        worst = max(worst, float(rel))
    assert worst <= 1.5 * 2.0 ** -50, worst


def test_silu_quant_on_a_dispatch_layout():
    # rows_in_use and padding come from a real PAD128 dispatch
    wl, x, idx, w = make_inputs("sweep_256", H=256)
    d = moe.dispatch(bf16_to_dev(x), to_dev(idx), to_dev(w), wl.E, wl.R, True, pad128=True)
    rows = d.recv_x.shape[0]
    I = 2048
    gu, _ = _silu_problem(rows, I, 11, pad_frac=0.0)
    act, sc = moe.silu_quant(bf16_to_dev(gu), d.recv_src, d.expert_offset[wl.E:])
    src = d.recv_src.cpu().numpy()
    act_ref, sc_ref = oracle.silu_quant(gu, src, int(d.expert_offset[wl.E].item()))
    np.testing.assert_array_equal(act.view(torch.uint8).cpu().numpy(), act_ref)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), sc_ref.view(np.uint32))


# ---- router top-k ---------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,fn,G,TG,renorm", [
    (128, 256, 8, "sigmoid", 1, 1, True),
    (128, 256, 8, "sigmoid", 8, 4, True),     # DeepSeek-V3-shaped group-limited routing
    (128, 384, 8, "softmax", 1, 1, True),
    (4096, 256, 8, "softmax", 1, 1, False),
    (1000, 64, 6, "softmax", 8, 3, True),
    (7, 1024, 32, "sigmoid", 32, 2, False),
    (33, 8, 2, "softmax", 2, 2, True),
    (300, 200, 8, "softmax", 8, 3, True),     # 25-expert groups straddle the lanes
])
def test_router_topk(T, E, k, fn, G, TG, renorm):
    l = np.random.default_rng(T + E).standard_normal((T, E)).astype(np.float32)
    l[0, 3] = l[0, 5] = l[0].max() + 1.0            # a tie: the lower id comes first
    ref_idx, ref_w = oracle.router_topk(l, k, score_fn=fn, n_group=G, topk_group=TG, renormalize=renorm)
    idx, w = moe.router_topk(to_dev(l), k, score_fn=fn, n_group=G, topk_group=TG, renormalize=renorm)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=2e-6, atol=1e-9)


@pytest.mark.parametrize("name,fn", [("tiny", "softmax"), ("dsv3_decode", "sigmoid")])
def test_router_feeds_dispatch_like_the_generator(name, fn):
    wl = WORKLOADS[name]
    logits = make_router_logits(wl).astype(np.float32)
    idx, w = moe.router_topk(to_dev(logits), wl.k, score_fn=fn)
    ref_idx, ref_w = oracle.router_topk(logits, wl.k, score_fn=fn)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=2e-6)


@pytest.mark.parametrize("E,G,TG,fn", [(256, 1, 1, "softmax"), (256, 8, 4, "sigmoid"), (96, 4, 2, "softmax"),
                                       (384, 1, 1, "sigmoid")])
def test_router_topk_ties_zeros_and_infinities(E, G, TG, fn):
    # few distinct logits, so most picks are decided by the lower-id rule; signed
    # zeros compare equal; -inf logits are the last choice
    rng = np.random.default_rng(E + G)
    T, k = 512, 8
    l = (rng.integers(-3, 4, size=(T, E)) * 0.5).astype(np.float32)
    l[rng.random((T, E)) < 0.3] = -0.0
    l[rng.random((T, E)) < 0.1] = -np.inf
    ref_idx, ref_w = oracle.router_topk(l, k, score_fn=fn, n_group=G, topk_group=TG, renormalize=True)
    idx, w = moe.router_topk(to_dev(l), k, score_fn=fn, n_group=G, topk_group=TG, renormalize=True)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=2e-6, atol=1e-9)


# ---- router feeding dispatch in one call ------------------------------------------------

@pytest.mark.parametrize("T,E,R,k,H,fn,G,TG,fp8,pad", [
    (128, 256, 8, 8, 7168, "sigmoid", 8, 4, True, False),   # DeepSeek-V3-shaped decode (one launch)
    (128, 384, 16, 8, 7168, "softmax", 1, 1, True, False),  # Kimi-K2-shaped: 12 logits per lane
    (16, 8, 2, 2, 256, "softmax", 1, 1, False, False),
    (1, 64, 4, 4, 1024, "sigmoid", 4, 2, False, False),     # one token
    (147, 256, 8, 8, 2048, "softmax", 1, 1, True, False),   # 148 CTAs: every SM
    (20, 128, 8, 6, 16384, "sigmoid", 1, 1, True, False),   # 2 chunks per warp
    (9, 32, 4, 8, 24576, "softmax", 1, 1, False, False),    # 4 chunks per warp
    (64, 256, 8, 8, 7168, "softmax", 1, 1, True, True),     # padding: router, then dispatch
    (3000, 256, 32, 8, 512, "softmax", 1, 1, True, True),   # tiled metadata path
])
def test_route_dispatch_equals_router_then_dispatch(T, E, R, k, H, fn, G, TG, fp8, pad):
    rng = np.random.default_rng(T + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    d, idx, w = moe.route_dispatch(bf16_to_dev(x), to_dev(logits), k, E, R, fp8, pad,
                                   score_fn=fn, n_group=G, topk_group=TG)
    assert moe.check() == 0
    ref_idx, ref_w = oracle.router_topk(logits, k, score_fn=fn, n_group=G, topk_group=TG)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=2e-6, atol=1e-9)
    d2 = moe.dispatch(bf16_to_dev(x), idx.clone(), w.clone(), E, R, fp8, pad)
    for a, b in [(d.expert_count, d2.expert_count), (d.expert_offset, d2.expert_offset),
                 (d.rank_offset, d2.rank_offset), (d.handle.slot, d2.handle.slot)]:
        np.testing.assert_array_equal(a.cpu().numpy(), b.cpu().numpy())
    n = int(d.expert_offset[E].item())
    np.testing.assert_array_equal(d.recv_src[:n].cpu().numpy(), d2.recv_src[:n].cpu().numpy())
    valid = d.recv_src[:n] >= 0
    np.testing.assert_array_equal(d.recv_x[:n][valid].view(torch.uint8).cpu().numpy(),
                                  d2.recv_x[:n][valid].view(torch.uint8).cpu().numpy())
    o = oracle.dispatch(x, ref_idx, E=E, R=R, fp8=fp8, pad128=pad)
    np.testing.assert_array_equal(d.handle.slot.cpu().numpy(), o["slot"])


def _graph_kernel_count(fn):
    """Kernel nodes of a CUDA graph captured around fn() (after one warm-up call)."""
    from cuda.bindings import driver as drv
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g):
        fn()
    graph = drv.CUgraph(g.raw_cuda_graph())
    _, _, n = drv.cuGraphGetNodes(graph, 0)
    _, nodes, n = drv.cuGraphGetNodes(graph, n)
    kinds = [drv.cuGraphNodeGetType(node)[1] for node in nodes[:n]]
    return sum(k == drv.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL for k in kinds)


def test_route_dispatch_repeats_on_the_same_buffers():
    # the dispatch kernel after the router reads x before the router has
    # finished: fresh logits each call must still give the oracle's choice and
    # dispatch, call after call and in a captured graph
    T, E, R, k, H = 128, 256, 8, 8, 7168
    rng = np.random.default_rng(41)
    xh = f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    x = bf16_to_dev(xh)
    cfg = moe.make_config(H, k, E, R, True, False)
    buf = moe.Buffers(cfg, T, "cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.check()
    for rep in range(3):
        logits = rng.standard_normal((T, E)).astype(np.float32)
        moe.route_dispatch_into(buf, x, to_dev(logits), idx, wt, score_fn="sigmoid")
        torch.cuda.synchronize()
        assert moe.check() == 0
        ref_idx, _ = oracle.router_topk(logits, k, score_fn="sigmoid")
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
        o = oracle.dispatch(xh, ref_idx, E=E, R=R, fp8=True, rows_cap=buf.rows_cap)
        np.testing.assert_array_equal(buf.slot.cpu().numpy(), o["slot"])
        valid = o["recv_src"] >= 0
        np.testing.assert_array_equal(buf.recv_x.view(torch.uint8).cpu().numpy()[valid], o["recv_x"][valid])
    ld = to_dev(rng.standard_normal((T, E)).astype(np.float32))
    assert _graph_kernel_count(lambda: moe.route_dispatch_into(buf, x, ld, idx, wt, score_fn="sigmoid")) == 2
    assert moe.check() == 0
