"""Pins of the oracle's sender-side (per-rank) partial combine.

"Enabling trillion-parameter models on AWS EFA", section "Avaliação": DeepEP
accumulates on the sending side to move less data, with possible precision
costs.  Each virtual rank sums a token's contributions from the experts it
hosts into one bf16 row; the token's home sums those rows.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from workloads import bf16_bits_to_f32, make_expert_out, make_inputs, random_problem


def _bf16_value(bits):
    return float(bf16_bits_to_f32(np.array([bits], np.uint16))[0])


def _nearest_bf16_exact(v: float) -> int:
    """Brute force: the bf16 bit pattern nearest to v (exact rationals), ties to even."""
    f = np.float32(v)
    base = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
    best = None
    for b in (base - 1, base, base + 1, base + 2):
        b &= 0xFFFF
        d = abs(Fraction(_bf16_value(b)) - Fraction(v))
        if best is None or d < best[0] or (d == best[0] and b % 2 == 0):
            best = (d, b)
    return best[1]


def test_partial_rounding_is_nearest_even_bf16():
    rng = np.random.default_rng(3)
    idx = np.zeros((1, 1), np.int32)
    slot = np.zeros((1, 1), np.int32)
    for _ in range(400):
        # one entry with weight w on a row of ones: the partial is bf16(w) exactly rounded
        w = float(rng.standard_normal() * 2.0 ** rng.integers(-8, 8))
        eo = np.full((1, 4), 0x3F80, np.uint16)  # 1.0
        o = oracle.combine_rank_partial(idx, slot, np.array([[w]], np.float32), eo, E=1, R=1)
        assert o["partial"][0, 0, 0] == _nearest_bf16_exact(float(np.float32(w)))


def test_partial_rounding_ties_go_to_even():
    # weights whose low 16 bits are exactly 0x8000 sit halfway between two bf16
    # values: the partial takes the one with an even last bit
    idx = np.zeros((1, 1), np.int32)
    slot = np.zeros((1, 1), np.int32)
    eo = np.full((1, 4), 0x3F80, np.uint16)  # 1.0
    for bits, want in [(0x3F808000, 0x3F80), (0x3F818000, 0x3F82), (0xBF808000, 0xBF80),
                       (0xBF818000, 0xBF82), (0x40A78000, 0x40A8), (0x3C008000, 0x3C00)]:
        w = np.array([[bits]], np.uint32).view(np.float32)
        o = oracle.combine_rank_partial(idx, slot, w, eo, E=1, R=1)
        assert o["partial"][0, 0, 0] == want == _nearest_bf16_exact(float(w[0, 0])), hex(bits)


def test_one_rank_equals_receiver_sum_rounded_once():
    x, idx, w = random_problem(4, 30, 64, 8, 4)
    d = oracle.dispatch(x, idx, E=8, R=1, fp8=False)
    eo = make_expert_out(make_inputs("tiny")[0], d["rows_cap"])[:, :64].copy()
    ref = oracle.combine(d["slot"], w, eo)
    o = oracle.combine_rank_partial(idx, d["slot"], w, eo, E=8, R=1)
    assert np.all(o["npart"] == 1)
    want = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(o["partial"][:, 0, :], want)


@pytest.mark.parametrize("E,R", [(8, 2), (16, 16), (256, 32)])
def test_ranks_per_token_and_error_bound(E, R):
    x, idx, w = random_problem(5, 40, 32, E, 8 if E >= 8 else 2)
    d = oracle.dispatch(x, idx, E=E, R=R, fp8=False)
    eo = make_expert_out(make_inputs("tiny")[0], d["rows_cap"])[:, :32].copy()
    exact = oracle.combine(d["slot"], w, eo)
    o = oracle.combine_rank_partial(idx, d["slot"], w, eo, E=E, R=R)
    k = idx.shape[1]
    for t in range(idx.shape[0]):
        ranks = idx[t] // (E // R)
        n = o["npart"][t]
        assert n == len(set(ranks.tolist())) <= min(k, R)
        first = list(dict.fromkeys(ranks.tolist()))       # order of first appearance
        np.testing.assert_array_equal(o["partial_rank"][t, :n], first)
    # each partial is within half a bf16 unit of its exact value, so the sum is within their total
    p = bf16_bits_to_f32(o["partial"]).astype(np.float64)
    half_ulp = np.where(p == 0, 0.0, np.exp2(np.floor(np.log2(np.abs(p) + 1e-300)) - 8))
    bound = half_ulp.sum(axis=1) * 1.0000001 + 1e-12
    assert np.all(np.abs(o["y"] - exact) <= bound)
