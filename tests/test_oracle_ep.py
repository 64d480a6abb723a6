"""The expert-parallel layout reading, checked against the single-GPU oracle.

"Enabling trillion-parameter models on AWS EFA", sections "Buffers de Envio e
Recebimento" and "Despacho e Combinação": ranks exchange per-expert counts, and
each sender writes its rows into a contiguous range of every peer's receive
buffer.  The layout adopted: rank d's buffer holds, expert by expert, the rows
from rank 0, then rank 1, ..., each in (token, k) order, each expert padded to
128 rows under PAD128.  Written out from the gathered counts, a sender's row is
  off_d(e) + sum_{s' < s} cnt[s'][e] + (rank of the entry among s's entries with e);
this must be the oracle's single-GPU dispatch of the concatenated batches, less
rank d's offset.
"""
import numpy as np
import pytest

import oracle
from workloads import random_problem


def _rows_from_counts(idx_by_rank, E, W, pad):
    El = E // W
    cnt = np.zeros((W, E), np.int64)
    for s, idx in enumerate(idx_by_rank):
        ok = (idx >= 0) & (idx < E)
        np.add.at(cnt[s], idx[ok], 1)
    tot = cnt.sum(0)
    seg = (tot + 127) // 128 * 128 if pad else tot
    off = np.zeros(E, np.int64)
    for d in range(W):                       # offsets restart at every rank's first expert
        off[d * El:(d + 1) * El] = np.concatenate([[0], np.cumsum(seg[d * El:(d + 1) * El])[:-1]])
    rows = []
    for s, idx in enumerate(idx_by_rank):
        before = cnt[:s].sum(0)
        seen = np.zeros(E, np.int64)
        r = np.full(idx.shape, -1, np.int64)
        for t in range(idx.shape[0]):
            for j in range(idx.shape[1]):
                e = idx[t, j]
                if 0 <= e < E:
                    r[t, j] = off[e] + before[e] + seen[e]
                    seen[e] += 1
        rows.append(r)
    return rows, tot, off


@pytest.mark.parametrize("W,E,k,Ts,pad", [(2, 8, 2, [5, 7], False), (4, 16, 3, [9, 0, 4, 11], True),
                                          (3, 6, 2, [20, 1, 13], True), (8, 64, 8, [16] * 8, False)])
def test_layout_from_counts_is_the_concatenated_dispatch(W, E, k, Ts, pad):
    batches = [random_problem(50 + s, T, 8, E, k, distinct=E >= k)[1] for s, T in enumerate(Ts)]
    batches[0] = batches[0].copy()
    if Ts[0]:
        batches[0][0, 0] = E                 # a bad id is dropped on both sides
    rows, tot, off = _rows_from_counts(batches, E, W, pad)
    IDX = np.concatenate(batches)
    X = np.zeros((IDX.shape[0], 8), np.uint16)
    o = oracle.dispatch(X, IDX, E=E, R=W, fp8=False, pad128=pad)
    El = E // W
    starts = np.cumsum([0] + Ts)
    for s in range(W):
        slot = o["slot"][starts[s]:starts[s + 1]]
        host = np.clip(batches[s], 0, E - 1) // El
        want = np.where(slot >= 0, slot - o["rank_offset"][host], -1)
        np.testing.assert_array_equal(rows[s], want)
    np.testing.assert_array_equal(tot, o["expert_count"])
    for d in range(W):
        np.testing.assert_array_equal(off[d * El:(d + 1) * El],
                                      o["expert_offset"][d * El:(d + 1) * El] - o["rank_offset"][d])
