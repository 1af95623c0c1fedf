"""Pins of the oracle's retrieval steps (projection, n-grams, hashing, gather)
against hand-worked cases, invariants and the birthday bound.  CPU only."""
import math

import numpy as np
import pytest

from oracle import engram_oracle as O
from hashed_gram_conditional_engram_b200 import synth
from tests.golden_io import rows as golden


def test_vocab_proj_golden():
    keys, want, vc = golden("vocab_proj.txt")
    proj, V_c = O.build_vocab_proj(np.array(keys, dtype=np.int64))
    assert proj.tolist() == want
    assert V_c == vc[0]


def test_vocab_proj_invariants_synthetic():
    # merge map of the tiny workload: 1,000 raw ids, 23% merged -> 770 ids
    w = synth.workload("tiny")
    keys = synth.merge_keys(np.random.default_rng(5), w.V, w.V_c)
    proj, V_c = O.build_vocab_proj(keys)
    assert V_c == 770 == w.V_c
    # same partition as an independent grouping by key (np.unique)
    _, inv = np.unique(keys, return_inverse=True)
    pairs = set(zip(proj.tolist(), inv.tolist()))
    assert len(pairs) == V_c                      # bijection between the two labelings
    # first occurrences are numbered 0, 1, 2, ... in raw id order
    seen, firsts = set(), []
    for p in proj.tolist():
        if p not in seen:
            seen.add(p)
            firsts.append(p)
    assert firsts == list(range(V_c))


def test_vocab_sizes_from_pages():
    # ~23% of a ~128k vocabulary merged (reportify.cn 技术创新与架构; deepseek.club 二.1 (1))
    assert synth.compressed_vocab(129280) == 99546
    assert synth.compressed_vocab(1000) == 770
    # 3-gram space "2x10^15" (deepseek.club 二.1 (1)) is the raw vocabulary cubed
    assert 2.0e15 <= 129280 ** 3 < 2.2e15


def test_ngrams_golden():
    g = golden("ngrams.txt")
    c = np.array([g[0]], dtype=np.int64)
    out = O.suffix_ngrams(c, pad=10)
    assert out[0].tolist() == g[1:]


def test_hash_golden():
    for order, P, m0, m1, m2, g0, g1, g2, want in golden("hash_cases.txt"):
        K = 1
        mult = np.array([[m0, m1, m2], [m0, m1, m2]], dtype=np.uint64)
        rows = np.array([P, P], dtype=np.int64)
        g = np.array([[g0, g1, g2]], dtype=np.int64)
        idx = O.hash_heads(g, mult, rows, K)
        assert int(idx[0, order - 2]) == want, (order, P, m0, m1, m2, g0, g1, g2)


def test_hash_range_and_determinism():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    proj, V_c = O.build_vocab_proj(inp["keys"])
    idx = O.hash_indices(proj, inp["ids"], inp["mult"], inp["rows"], w.K, V_c)
    assert idx.shape == (w.B, w.T, w.J)
    assert idx.min() >= 0 and (idx < inp["rows"][None, None, :]).all()
    idx2 = O.hash_indices(proj.copy(), inp["ids"].copy(), inp["mult"].copy(), inp["rows"], w.K, V_c)
    assert np.array_equal(idx, idx2)


def test_hash_depends_only_on_suffix():
    # the slot of position t depends on c_t, c_{t-1} (and c_{t-2} for 3-grams) only
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    proj, V_c = O.build_vocab_proj(inp["keys"])
    ids = inp["ids"].copy()
    base = O.hash_indices(proj, ids, inp["mult"], inp["rows"], w.K, V_c)
    ids[0, 20] = (ids[0, 20] + 1) % w.V
    while proj[ids[0, 20]] == proj[inp["ids"][0, 20]]:
        ids[0, 20] = (ids[0, 20] + 1) % w.V
    pert = O.hash_indices(proj, ids, inp["mult"], inp["rows"], w.K, V_c)
    changed = np.any(base != pert, axis=-1)[0]
    assert not changed[:20].any() and not changed[23:].any()
    # 2-gram heads see t and t+1, 3-gram heads t..t+2
    assert np.any(base[0, 22, w.K:] != pert[0, 22, w.K:])
    assert np.array_equal(base[0, 22, :w.K], pert[0, 22, :w.K])


def test_hash_birthday_bound():
    """n distinct n-grams hashed into P slots: the expected fraction of keys that
    share their slot with another key is 1 - (1 - 1/P)^(n-1)."""
    rng = np.random.default_rng(11)
    P, n, trials, V_c = 1009, 64, 3000, 770
    rows = np.array([P, P], dtype=np.int64)
    fr = np.empty(trials)
    for tr in range(trials):
        mult = synth.hash_multipliers(1000 + tr, 2)
        flat = rng.choice(V_c * V_c, size=n, replace=False)
        g = np.stack([flat // V_c, flat % V_c, np.zeros(n, np.int64)], axis=-1)
        slots = O.hash_heads(g, mult, rows, 1)[:, 0]
        cnt = np.bincount(slots, minlength=P)
        fr[tr] = np.sum(cnt[slots] > 1) / n
    expect = 1.0 - (1.0 - 1.0 / P) ** (n - 1)
    se = fr.std(ddof=1) / math.sqrt(trials)
    assert abs(fr.mean() - expect) < 3.0 * se + 1e-4, (fr.mean(), expect, se)


@pytest.mark.parametrize("order", [2, 3])
def test_hash_uniform_bruteforce(order):
    """All V_c^order n-grams of a tiny vocabulary: each head's slot counts are
    uniform by a chi-square test (df = P - 1)."""
    V_c, P = 40, 101
    grid = np.stack(np.meshgrid(*[np.arange(V_c)] * order, indexing="ij"), -1).reshape(-1, order)
    g = np.concatenate([grid, np.zeros((grid.shape[0], 3 - order), np.int64)], axis=1)
    K = 4
    mult = synth.hash_multipliers(99, 2 * K)
    rows = np.full(2 * K, P, dtype=np.int64)
    idx = O.hash_heads(g, mult, rows, K)
    heads = range(0, K) if order == 2 else range(K, 2 * K)
    n = g.shape[0]
    for j in heads:
        cnt = np.bincount(idx[:, j], minlength=P)
        exp = n / P
        chi2 = float(np.sum((cnt - exp) ** 2 / exp))
        assert chi2 < (P - 1) + 6.0 * math.sqrt(2 * (P - 1)), (j, chi2)
    # the heads are independent: two heads never give the same slot sequence
    h0 = list(heads)[0]
    h1 = list(heads)[1]
    assert np.mean(idx[:, h0] == idx[:, h1]) < 3.0 / P


def test_gather_decodes_to_indices():
    # tables whose entries encode (head, slot, column): the gathered vector must
    # decode back to the requested slot of each head, in head order
    J, D_h, P = 4, 16, 1009
    tables = [np.array([[j * 1e6 + s * 100 + c for c in range(D_h)] for s in range(P)],
                       dtype=np.float64) for j in range(J)]
    rng = np.random.default_rng(3)
    idx = rng.integers(0, P, size=(5, 7, J)).astype(np.int32)
    e = O.gather(idx, tables)
    assert e.shape == (5, 7, J * D_h)
    for j in range(J):
        seg = e[..., j * D_h:(j + 1) * D_h]
        assert np.array_equal(seg[..., 0] // 1e6, np.full(idx.shape[:2], j))
        assert np.array_equal((seg[..., 0] % 1e6) // 100, idx[..., j])
        assert np.array_equal(seg[..., 3] - seg[..., 0], np.full(idx.shape[:2], 3.0))


def test_decode_state_matches_prefill():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    proj, V_c = O.build_vocab_proj(inp["keys"])
    ids = np.random.default_rng(4).integers(0, w.V, size=(3, 9)).astype(np.int32)
    full = O.hash_indices(proj, ids, inp["mult"], inp["rows"], w.K, V_c)
    state = np.full((3, 2), V_c, dtype=np.int32)
    for t in range(9):
        idx_t, state = O.hash_indices_decode(proj, ids[:, t], state, inp["mult"], inp["rows"], w.K)
        assert np.array_equal(idx_t, full[:, t])


def test_out_of_range_id_is_an_error():
    proj = np.arange(10, dtype=np.int32)
    with pytest.raises(ValueError):
        O.compress(proj, np.array([3, 10]))
    with pytest.raises(ValueError):
        O.compress(proj, np.array([-1]))


def test_workload_table_sizes_from_pages():
    # Engram-27B: 5.7B memory parameters (reportify.cn 性能提升; deepseek.club 三.2)
    w2 = synth.workload("layer27b")
    assert abs(w2.table_params() - 5.7e9) < 0.01e9
    assert all(synth._is_prime(p) for p in w2.rows)
    # scaling experiment up to +13B parameters (gitcode.csdn.net blog, 实际效果)
    w4 = synth.workload("decode")
    assert abs(w4.table_params() - 13.0e9) < 0.01e9
    # 100B-parameter table offloaded to host DRAM (deepseek.club 三.4)
    w5 = synth.workload("hosttable")
    assert abs(w5.table_params() - 100e9) < 0.01e9
