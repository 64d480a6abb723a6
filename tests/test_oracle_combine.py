"""Pins of the oracle's combine: the routing-weighted sum of the experts' rows.

"Enabling trillion-parameter models on AWS EFA" (sections "Introdução" and
"Despacho e Combinação") and "Lower latency and higher throughput with
multi-node DeepSeek deployment" (section "Paralelismo de Especialistas") define
combine as the weighted sum of each token's processed rows.  These tests check
the oracle with closed forms and a linear-algebra restatement.
"""
import numpy as np
import pytest

import oracle
from workloads import bf16_bits_to_f32, make_expert_out, make_inputs, random_problem

TOL_ABS, TOL_REL = 1e-2, 4e-3


def _decode_e4m3(c):
    c = np.asarray(c, np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    f, m = (c >> 3) & 0xF, c & 0x7
    return s * np.where(f == 0, m * 2.0 ** -9, (1 + m / 8.0) * np.exp2(f - 7.0))


def test_identity_experts_return_weighted_input():
    # tiny workload: expert_out = the dispatched bf16 rows, so y = x * sum_j w_j
    w, x, idx, wts = make_inputs("tiny")
    d = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=False)
    y = oracle.combine(d["slot"], wts, d["recv_x"])
    xf = bf16_bits_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(y, xf * wts.astype(np.float64).sum(1, keepdims=True), rtol=1e-12, atol=0)
    assert np.all(np.abs(wts.sum(1) - 1) < 1e-6)


def test_one_hot_weights_select_a_row_exactly():
    x, idx, _ = random_problem(3, T=20, H=64, E=8, k=4)
    d = oracle.dispatch(x, idx, E=8, R=2, fp8=False)
    eo = make_expert_out(make_inputs("tiny")[0], d["rows_cap"])[:, :64].copy()
    eo = np.ascontiguousarray(eo)
    for j in range(4):
        w = np.zeros((20, 4), np.float32)
        w[:, j] = 1.0
        y = oracle.combine(d["slot"], w, eo)
        np.testing.assert_array_equal(y, bf16_bits_to_f32(eo[d["slot"][:, j]]).astype(np.float64))


def test_matches_sparse_matrix_product():
    # y = A @ expert_out, with A[t, slot[t,j]] = w[t,j]: a library matmul, other order
    x, idx, wts = random_problem(4, T=50, H=96, E=10, k=3, distinct=False)
    d = oracle.dispatch(x, idx, E=10, R=5, fp8=False)
    rng = np.random.default_rng(9)
    eo = (rng.integers(0, 0x7F7F, size=(d["rows_cap"], 96)) & 0x3FFF).astype(np.uint16)
    A = np.zeros((50, d["rows_cap"]))
    for t in range(50):
        for j in range(3):
            A[t, d["slot"][t, j]] += wts[t, j]
    ref = A @ bf16_bits_to_f32(eo).astype(np.float64)
    y = oracle.combine(d["slot"], wts, eo)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_linear_in_weights():
    x, idx, w1 = random_problem(5, T=30, H=32, E=6, k=2)
    _, _, w2 = random_problem(6, T=30, H=32, E=6, k=2)
    d = oracle.dispatch(x, idx, E=6, R=3, fp8=False)
    eo = d["recv_x"]
    y12 = oracle.combine(d["slot"], w1 + w2, eo)
    y1 = oracle.combine(d["slot"], w1, eo)
    y2 = oracle.combine(d["slot"], w2, eo)
    # w1 + w2 is rounded to binary32, so compare against that sum's effect loosely
    np.testing.assert_allclose(y12, y1 + y2, rtol=1e-6, atol=1e-6)


def test_dropped_entries_contribute_nothing():
    x, idx, wts = random_problem(7, T=8, H=16, E=4, k=2)
    d = oracle.dispatch(x, idx, E=4, R=2, fp8=False)
    slot = d["slot"].copy()
    slot[:, 1] = -1
    y = oracle.combine(slot, wts, d["recv_x"])
    xf = bf16_bits_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(y, xf * wts[:, :1].astype(np.float64), rtol=1e-12, atol=0)


def test_sampled_tokens_match_full():
    x, idx, wts = random_problem(8, T=40, H=32, E=8, k=4)
    d = oracle.dispatch(x, idx, E=8, R=2, fp8=False)
    full = oracle.combine(d["slot"], wts, d["recv_x"])
    toks = [39, 0, 17, 17]
    np.testing.assert_array_equal(oracle.combine(d["slot"], wts, d["recv_x"], tokens=toks), full[toks])


def test_fp8_identity_expert_within_quantisation_error():
    # an expert that dequantises its fp8 input returns x up to the e4m3 grid error
    w, x, idx, wts = make_inputs("dsv3_decode", T=8)
    d = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=True)
    deq = _decode_e4m3(d["recv_x"]) * np.repeat(d["recv_scale"].astype(np.float64), 128, axis=1)
    y = np.zeros((w.T, w.H))
    for t in range(w.T):
        for j in range(w.k):
            y[t] += wts[t, j] * deq[d["slot"][t, j]]
    xf = bf16_bits_to_f32(x).astype(np.float64)
    amax = np.abs(xf.reshape(w.T, -1, 128)).max(-1)
    # per element |code*scale - x| <= half the widest e4m3 step (32, on [256, 448]) times
    # the scale amax/448; the weights sum to 1, so the same bound holds for y
    bound = np.repeat(amax / 448.0 * 16.0, 128, axis=1) * (1 + 1e-6)
    assert np.all(np.abs(y - xf * wts.sum(1, keepdims=True)) <= bound)


@pytest.mark.parametrize("name", ["tiny", "dsv3_decode"])
def test_tolerance_rule_accepts_bf16_rounding(name):
    # rounding the fp64 result to bf16 (what the GPU returns) stays inside the stated rule
    w, x, idx, wts = make_inputs(name)
    d = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=w.fp8)
    eo = d["recv_x"] if w.identity_experts else make_expert_out(w, d["rows_cap"])
    y = oracle.combine(d["slot"], wts, eo)
    import torch
    yb = torch.from_numpy(y).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.all(np.abs(yb - y) <= TOL_ABS + TOL_REL * np.abs(y))
