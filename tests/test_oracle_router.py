"""Pins of the oracle's router top-k.

"Lower latency and higher throughput with multi-node DeepSeek deployment",
section "Roteador MoE": one top-k with index tracking serves every MoE model;
plain top-k is group-limited top-k with one group.
"""
import numpy as np
import pytest

import oracle
from workloads import WORKLOADS, make_router_logits, make_routing


def _logits(seed, T, E):
    return np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)


@pytest.mark.parametrize("score_fn", ["softmax", "sigmoid"])
def test_one_group_is_a_stable_descending_sort(score_fn):
    l = _logits(1, 64, 96)
    l[5, 10] = l[5, 20] = l[5].max() + 1.0           # a tie at the top: lower id first
    idx, _ = oracle.router_topk(l, 6, score_fn=score_fn)
    ref = np.argsort(-l, axis=1, kind="stable")[:, :6]
    np.testing.assert_array_equal(idx, ref)


def test_weights_closed_forms():
    l = _logits(2, 50, 32).astype(np.float64)
    idx, w = oracle.router_topk(l, 4, score_fn="softmax", renormalize=True)
    sel = np.take_along_axis(l, idx, 1)
    e = np.exp(sel - sel.max(1, keepdims=True))
    np.testing.assert_allclose(w, e / e.sum(1, keepdims=True), rtol=1e-6)
    idx, w = oracle.router_topk(l, 4, score_fn="softmax", renormalize=False)
    p = np.exp(l - l.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, 1), rtol=1e-6)
    idx, w = oracle.router_topk(l, 4, score_fn="sigmoid", renormalize=False)
    np.testing.assert_allclose(w, 1 / (1 + np.exp(-np.take_along_axis(l, idx, 1))), rtol=1e-6)


def test_group_limited_invariants():
    E, G, TG, k = 64, 8, 3, 6
    l = _logits(3, 200, E)
    idx, w = oracle.router_topk(l, k, score_fn="sigmoid", n_group=G, topk_group=TG)
    gsize = E // G
    for t in range(l.shape[0]):
        gmax = l[t].reshape(G, gsize).max(1)
        kept = set(np.argsort(-gmax, kind="stable")[:TG].tolist())
        chosen = idx[t].tolist()
        assert all(e // gsize in kept for e in chosen)
        assert len(set(chosen)) == k
        cand = [e for e in range(E) if e // gsize in kept and e not in chosen]
        assert max(l[t, cand]) <= min(l[t, chosen])             # nothing better was left out
        assert list(l[t, chosen]) == sorted(l[t, chosen], reverse=True)
        np.testing.assert_allclose(w[t].sum(), 1.0, rtol=1e-6)


def test_group_ties_keep_the_lower_group():
    # groups 1 and 3 share the largest maximum; with one group kept it is group 1
    E, G = 16, 4
    l = np.full((2, E), -1.0, np.float32)
    l[:, 4:8] = [0.5, 2.0, 0.1, 0.2]      # group 1
    l[:, 12:16] = [2.0, 1.5, 1.4, 1.3]    # group 3: same maximum, better runners-up
    idx, _ = oracle.router_topk(l, 2, score_fn="softmax", n_group=G, topk_group=1)
    np.testing.assert_array_equal(idx, [[5, 4], [5, 4]])
    idx, _ = oracle.router_topk(l, 3, score_fn="sigmoid", n_group=G, topk_group=2)
    np.testing.assert_array_equal(idx, [[5, 12, 13], [5, 12, 13]])


def test_brute_force_small_group_limited():
    # every choice of groups: the chosen set maximises the sum of logits among
    # sets drawn from the best topk_group groups (by group maximum)
    import itertools
    E, G, TG, k = 8, 4, 2, 3
    rng = np.random.default_rng(4)
    for _ in range(300):
        l = rng.standard_normal((1, E)).astype(np.float32)
        idx, _ = oracle.router_topk(l, k, n_group=G, topk_group=TG)
        gmax = l[0].reshape(G, E // G).max(1)
        groups = sorted(range(G), key=lambda g: (-gmax[g], g))[:TG]
        cand = [e for e in range(E) if e // (E // G) in groups]
        best = max(itertools.combinations(cand, k), key=lambda c: (sorted(l[0, list(c)], reverse=True)))
        assert sorted(idx[0].tolist()) == sorted(best)


@pytest.mark.parametrize("name,score_fn", [("tiny", "softmax"), ("dsv3_decode", "sigmoid")])
def test_reproduces_the_workload_generator(name, score_fn):
    w = WORKLOADS[name]
    logits = make_router_logits(w)
    idx, wts = oracle.router_topk(logits.astype(np.float32), w.k, score_fn=score_fn)
    ref_idx, ref_w = make_routing(w)
    np.testing.assert_array_equal(idx, ref_idx)
    np.testing.assert_allclose(wts, ref_w, rtol=2e-6)
