"""Pins of the oracle's dispatch: counts, offsets, slots and payload.

The dispatch is a stable counting sort of the T*k routing entries by expert id,
followed by a row copy ("Enabling trillion-parameter models on AWS EFA",
sections "Buffers de Envio e Recebimento" and "Despacho e Combinação": counts
per expert, their cumulative sum as offsets, contiguous packing).  These tests
check the oracle against properties and routines it does not use itself.
"""
import itertools

import numpy as np
import pytest

import oracle
from workloads import WORKLOADS, make_inputs, random_problem


def _check_invariants(o, idx, E, R, pad128, x=None, fp8=False):
    T, k = idx.shape
    S = T * k
    cnt, off, roff = o["expert_count"], o["expert_offset"], o["rank_offset"]
    slot, src = o["slot"], o["recv_src"]
    valid = (idx >= 0) & (idx < E)
    # counts: library histogram of the valid entries, summing to T*k when all are valid
    np.testing.assert_array_equal(cnt, np.bincount(idx[valid].ravel(), minlength=E))
    assert cnt.sum() == valid.sum()
    # offsets: textbook exclusive scan of the (padded) counts
    seg = (cnt + 127) // 128 * 128 if pad128 else cnt
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(seg)]))
    if pad128:
        assert np.all(off % 128 == 0)
    # ranks own contiguous expert ranges, so rank offsets are a subsequence
    np.testing.assert_array_equal(roff, off[:: E // R])
    # every valid (t, j) lands exactly once, inside its expert's segment
    flat = slot.ravel()
    kept = flat[valid.ravel()]
    assert np.all(kept >= 0)
    assert len(np.unique(kept)) == kept.size
    e_of = idx.ravel()[valid.ravel()]
    assert np.all(kept >= off[e_of]) and np.all(kept < off[e_of] + cnt[e_of])
    ent = np.nonzero(valid.ravel())[0]
    np.testing.assert_array_equal(src[kept], ent)
    # rows with no entry are -1, and there are exactly (rows_cap - kept) of them
    assert np.sum(src == -1) == src.size - kept.size
    # inside a segment, sources increase strictly: (token, k) order
    for e in range(E):
        s = src[off[e]:off[e] + cnt[e]]
        assert np.all(np.diff(s) > 0)
    if x is not None and not fp8:
        for t in range(T):
            for j in range(k):
                if slot[t, j] >= 0:
                    assert np.array_equal(o["recv_x"][slot[t, j]], x[t])


@pytest.mark.parametrize("name", ["tiny", "dsv3_decode", "kimi_decode"])
def test_invariants_on_workloads(name):
    w, x, idx, _ = make_inputs(name)
    o = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=w.fp8, pad128=w.pad128)
    assert o["err"] == 0
    assert o["expert_count"].sum() == w.T * w.k
    _check_invariants(o, idx, w.E, w.R, w.pad128, x, w.fp8)


def test_invariants_sweep_pad128_small_H():
    # the T=256 sweep's routing with a narrow hidden size keeps the test quick
    w, x, idx, _ = make_inputs("sweep_256", H=256)
    o = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=True, pad128=True)
    _check_invariants(o, idx, w.E, w.R, True)
    assert o["expert_offset"][-1] <= o["rows_cap"]


def test_prefill_zipf_routing_small_H():
    w, x, idx, _ = make_inputs("prefill_zipf", H=64)
    o = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=False)
    _check_invariants(o, idx, w.E, w.R, False, x)
    # the Zipf draw is skewed: the busiest expert takes most tokens
    assert o["expert_count"].max() > w.T // 2


@pytest.mark.parametrize("seed", range(4))
def test_equals_stable_argsort(seed):
    x, idx, _ = random_problem(seed, T=37, H=16, E=12, k=3, distinct=False)
    o = oracle.dispatch(x, idx, E=12, R=3, fp8=False)
    # library special case: a stable argsort by expert id lists entries in slot order
    np.testing.assert_array_equal(o["recv_src"], np.argsort(idx.ravel(), kind="stable"))


def _definition_by_expert(idx, E, pad128, rows_cap):
    """Independent statement: for each expert in turn, list its (t, j) entries in
    lexicographic order and give them consecutive rows from the running offset."""
    T, k = idx.shape
    slot = -np.ones((T, k), np.int64)
    src = -np.ones(rows_cap, np.int64)
    row = 0
    for e in range(E):
        mine = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e]
        for n, (t, j) in enumerate(mine):
            slot[t, j] = row + n
            src[row + n] = t * k + j
        row += (len(mine) + 127) // 128 * 128 if pad128 else len(mine)
    return slot, src


def test_brute_force_all_routings_distinct():
    E, k = 4, 2
    pairs = [p for p in itertools.permutations(range(E), k)]
    x = np.arange(3 * 8, dtype=np.uint16).reshape(3, 8)
    for T in (1, 2, 3):
        for combo in itertools.product(pairs, repeat=T):
            idx = np.array(combo, np.int32).reshape(T, k)
            for pad in (False, True):
                o = oracle.dispatch(x[:T], idx, E=E, R=2, fp8=False, pad128=pad)
                s_ref, src_ref = _definition_by_expert(idx, E, pad, o["rows_cap"])
                np.testing.assert_array_equal(o["slot"], s_ref)
                np.testing.assert_array_equal(o["recv_src"], src_ref)


def test_brute_force_all_routings_with_duplicates():
    E, k, T = 3, 2, 2
    x = np.arange(T * 8, dtype=np.uint16).reshape(T, 8)
    for flat in itertools.product(range(E), repeat=T * k):
        idx = np.array(flat, np.int32).reshape(T, k)
        o = oracle.dispatch(x, idx, E=E, R=1, fp8=False)
        s_ref, src_ref = _definition_by_expert(idx, E, False, o["rows_cap"])
        np.testing.assert_array_equal(o["slot"], s_ref)
        np.testing.assert_array_equal(o["recv_src"], src_ref)
        _check_invariants(o, idx, E, 1, False, x)


def test_bad_index_is_dropped_and_flagged():
    x, idx, _ = random_problem(1, T=10, H=8, E=6, k=2)
    idx = idx.copy()
    idx[3, 1] = 6
    idx[7, 0] = -2
    o = oracle.dispatch(x, idx, E=6, R=2, fp8=False)
    assert o["err"] == oracle.BAD_INDEX
    assert o["slot"][3, 1] == -1 and o["slot"][7, 0] == -1
    assert o["expert_count"].sum() == 18
    _check_invariants(o, idx, 6, 2, False, x)


@pytest.mark.parametrize("bad", [-1, 4, 5, 2**31 - 1, -2**31])
def test_each_out_of_range_id_alone_is_flagged(bad):
    x, idx, _ = random_problem(9, T=6, H=8, E=4, k=2)
    idx = idx.copy()
    idx[2, 0] = bad
    o = oracle.dispatch(x, idx, E=4, R=1, fp8=False)
    assert o["err"] == oracle.BAD_INDEX
    assert o["slot"][2, 0] == -1 and o["expert_count"].sum() == 11


def test_capacity_overflow_is_dropped_and_flagged():
    x, idx, _ = random_problem(2, T=10, H=8, E=4, k=2)
    o = oracle.dispatch(x, idx, E=4, R=2, fp8=False, rows_cap=15)
    assert o["err"] == oracle.CAPACITY
    full = oracle.dispatch(x, idx, E=4, R=2, fp8=False)
    keep = full["slot"] < 15
    np.testing.assert_array_equal(o["slot"][keep], full["slot"][keep])
    assert np.all(o["slot"][~keep] == -1)
    np.testing.assert_array_equal(o["recv_src"], full["recv_src"][:15])


def test_empty_batch():
    x = np.zeros((0, 128), np.uint16)
    idx = np.zeros((0, 8), np.int32)
    o = oracle.dispatch(x, idx, E=16, R=4, fp8=True, pad128=True)
    assert o["err"] == 0 and o["rows_cap"] == 0
    assert np.all(o["expert_count"] == 0) and np.all(o["expert_offset"] == 0)


def _max_padded_rows(S, E):
    """Largest sum of per-expert counts rounded up to 128 over all ways to split S among E experts."""
    best = 0
    for c in itertools.product(range(S + 1), repeat=E):
        if sum(c) == S:
            best = max(best, sum((n + 127) // 128 * 128 for n in c))
    return best


def test_rows_capacity_is_the_worst_case():
    for S in range(0, 9):
        for E in (1, 2, 3, 4):
            for k in (1, S) if S else (1,):
                if S % k:
                    continue
                worst = _max_padded_rows(S, E)
                cap = oracle.rows_capacity(S // k, k, E, True)
                assert worst <= cap < worst + 128 and cap % 128 == 0
                assert oracle.rows_capacity(S // k, k, E, False) == S


def test_fp8_payload_matches_per_token_quantiser():
    w, x, idx, _ = make_inputs("dsv3_decode", T=16)
    o = oracle.dispatch(x, idx, E=w.E, R=w.R, fp8=True)
    for t in range(16):
        codes, scales = oracle.quantise_row_fp8(x[t])
        for j in range(w.k):
            s = o["slot"][t, j]
            np.testing.assert_array_equal(o["recv_x"][s], codes)
            np.testing.assert_array_equal(o["recv_scale"][s], scales)
    assert o["recv_scale"].shape[1] == w.H // 128  # (M, K) activation -> M x ceil(K/128) scales


def test_workload_table_shapes():
    for name, w in WORKLOADS.items():
        assert w.E % w.R == 0
        if w.fp8:
            assert w.H % 128 == 0


@pytest.mark.parametrize("fp8,pad128,threads", [(True, True, 4), (False, False, 3), (True, False, 8)])
def test_parallel_runner_is_bitwise_the_serial_oracle(fp8, pad128, threads):
    # the host-thread split used for the all-cores CPU baseline changes nothing
    from workloads import random_problem
    x, idx, w = random_problem(21, 301, 256, 16, 4)
    a = oracle.dispatch(x, idx, E=16, R=4, fp8=fp8, pad128=pad128)
    b = oracle.dispatch_parallel(x, idx, E=16, R=4, fp8=fp8, pad128=pad128, threads=threads)
    for key in ("recv_x", "recv_scale", "expert_count", "expert_offset", "rank_offset", "recv_src", "slot"):
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)
    assert a["err"] == b["err"]
    eo = a["recv_x"] if not fp8 else np.resize(x, (a["rows_cap"], 256))
    np.testing.assert_array_equal(oracle.combine(a["slot"], w, eo), oracle.combine_parallel(a["slot"], w, eo, threads))
