"""Pins of the oracle's hot-row ranking (the contents of an HBM cache in front
of a host-memory table) and of the gather's zero rows for invalid slots:
hand-worked cases, a brute-force count on small inputs, and invariants.
CPU only."""
from collections import Counter

import numpy as np

from oracle import engram_oracle as O


def test_hot_rows_hand_worked():
    # two heads of 5 and 7 rows: head 1's slot s is packed row 5 + s
    rows = [5, 7]
    idx = np.array([[0, 3],
                    [0, 3],
                    [4, 3],
                    [4, 0],
                    [-1, 6],
                    [0, 7],    # slot 7 is outside head 1's 7 rows: no row
                    [2, 6]], dtype=np.int32)
    # counts: row 0 x3, row 8 (head 1 slot 3) x3, row 4 x2, row 11 (slot 6) x2,
    # row 5 (slot 0) x1, row 2 x1
    top, n = O.hot_rows(idx, rows, 10)
    assert n == 6
    assert top.tolist() == [0, 8, 4, 11, 2, 5, -1, -1, -1, -1]
    top3, n3 = O.hot_rows(idx, rows, 3)
    assert n3 == 3 and top3.tolist() == [0, 8, 4]
    top0, n0 = O.hot_rows(idx, rows, 0)
    assert n0 == 0 and top0.size == 0


def _brute_force(idx, rows, C):
    """Count with a Python dict, then repeatedly take the best remaining row."""
    base = [sum(rows[:j]) for j in range(len(rows))]
    cnt = Counter()
    for tok in idx.reshape(-1, len(rows)).tolist():
        for j, s in enumerate(tok):
            if 0 <= s < rows[j]:
                cnt[base[j] + s] += 1
    left = dict(cnt)
    out = []
    while left and len(out) < C:
        best = None
        for r, c in left.items():
            if best is None or c > left[best] or (c == left[best] and r < best):
                best = r
        out.append(best)
        del left[best]
    return out + [-1] * (C - len(out)), min(C, len(cnt))


def test_hot_rows_matches_brute_force():
    rng = np.random.default_rng(11)
    for trial in range(20):
        J = int(rng.choice([4, 8]))
        rows = [int(x) for x in rng.integers(3, 40, J)]
        n_tok = int(rng.integers(0, 60))
        # skewed slots with ties, invalid -1 and out-of-range entries mixed in
        idx = np.stack([np.minimum(rng.zipf(1.6, n_tok) - 1, rows[j] + 2) for j in range(J)], -1)
        idx = np.where(rng.random(idx.shape) < 0.1, -1, idx).astype(np.int32)
        for C in (0, 1, 5, 200):
            top, n = O.hot_rows(idx, rows, C)
            want, wn = _brute_force(idx, rows, C)
            assert top.tolist() == want and n == wn, (trial, C)


def test_hot_rows_invariants():
    rng = np.random.default_rng(3)
    rows = [101, 103, 107, 109]
    idx = (rng.zipf(1.3, (500, 4)) % 100).astype(np.int32)
    top, n = O.hot_rows(idx, rows, 1000)
    base = np.array([0, 101, 204, 311])
    packed = (base[None, :] + idx).ravel()
    counts = Counter(packed.tolist())
    got = top[:n].tolist()
    assert sorted(got) == sorted(counts)          # every addressed row, once
    assert all(counts[a] >= counts[b] for a, b in zip(got, got[1:]))  # non-increasing
    assert sum(counts[r] for r in got) == idx.size  # the counts cover every pair
    assert (top[n:] == -1).all()


def test_gather_zero_rows_for_invalid_slots():
    tables = [np.arange(12, dtype=np.float32).reshape(3, 4) + 100 * j for j in range(2)]
    idx = np.array([[2, -1], [-1, 0]], dtype=np.int32)
    e = O.gather(idx, tables)
    assert e.tolist() == [[8, 9, 10, 11, 0, 0, 0, 0],
                          [0, 0, 0, 0, 100, 101, 102, 103]]


def test_history_ids_share_the_batch_vocabulary_permutation():
    """More text of the host-table workload's distribution (the history a
    cache is ranked on) maps ranks through the batch's own permutation:
    replaying the batch's draws with it reproduces the batch exactly."""
    from hashed_gram_conditional_engram_b200 import synth
    w = synth.workload("hosttable")
    ids, _ = synth.host_ids_keys(w)
    perm = synth.host_ids_perm(w)
    again = synth.zipf_ids(np.random.default_rng(w.seed), w.V, 1.1, w.N * w.steps, perm=perm)
    assert np.array_equal(again.reshape(ids.shape), ids)
