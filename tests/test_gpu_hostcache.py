"""Parity of the HBM cache of hot host-table rows with the oracle.

The ranking (engram_hostcache_rank) equals the oracle's hot_rows bit for bit;
the fill builds the row -> slot map and copies the rows exactly; the cached
gather (engram_forward_hostcache) returns e bit-identical to the oracle's
gather whatever the cache holds (empty, partial, every row), with the count
of (token, head) pairs read from host memory equal to the oracle's."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O
from tests.engram_cases import bf16_bits, dev

pytestmark = pytest.mark.gpu


def _ws(nbytes):
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device="cuda")


def _skewed_idx(rng, n_tok, rows, p_invalid=0.02):
    """Zipf(1.2)-skewed slots per head (frequent rows shared by many tokens),
    a few -1 slots."""
    idx = np.stack([(rng.zipf(1.2, n_tok) - 1) % P for P in rows], -1)
    idx = np.where(rng.random(idx.shape) < p_invalid, -1, idx)
    return idx.astype(np.int32)


@pytest.mark.parametrize("n_tok,C", [(3000, 0), (3000, 7), (3000, 500), (3000, 100000),
                                     (1, 3), (0, 4)])
def test_hostcache_rank_matches_oracle(n_tok, C):
    rng = np.random.default_rng(n_tok + C)
    K, D_h = 4, 32
    rows = synth.primes_at_most(4001, 2 * K)
    idx = _skewed_idx(rng, n_tok, rows)
    cfg = eg.make_cfg(K, D_h, 256, 1, 1000, 770, eg.BF16, rows, np.ones((2 * K, 3), np.uint64))
    nb = eg.engram_workspace_size(cfg, eg.WS_HOSTCACHE_RANK, n_tok)
    out = torch.full((max(C, 1),), 7, dtype=torch.int64, device="cuda")
    n_out = torch.full((1,), -5, dtype=torch.int32, device="cuda")
    eg.engram_hostcache_rank(cfg, dev(idx) if n_tok else None, n_tok, C, out, n_out, _ws(nb), nb)
    want, wn = O.hot_rows(idx, rows, C)
    assert int(n_out.item()) == wn
    assert out[:C].cpu().numpy().tolist() == want.tolist()
    assert eg.engram_get_status() == 0


def _host_table(rng, rows, D_h, dtype):
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    if dtype == eg.BF16:
        tb = [synth.to_bf16_bits(t) for t in tables]
        host = torch.from_numpy(np.concatenate([t.reshape(-1) for t in tb]).view(np.int16))
    else:
        tb = tables
        host = torch.from_numpy(np.concatenate([t.reshape(-1) for t in tb]))
    return tb, host.pin_memory()


@pytest.mark.parametrize("dtype", [eg.BF16, eg.F32])
@pytest.mark.parametrize("cache_rows", ["none", "hot", "all"])
def test_hostcache_gather_bit_exact(dtype, cache_rows):
    rng = np.random.default_rng(5 + dtype)
    K, D_h = 4, 32 if dtype == eg.BF16 else 16
    rows = synth.primes_at_most(2003, 2 * K)
    J = 2 * K
    tb, host = _host_table(rng, rows, D_h, dtype)
    cfg = eg.make_cfg(K, D_h, 256, 1, 1000, 770, dtype, rows, np.ones((J, 3), np.uint64))
    total = eg.engram_table_rows(cfg)
    assert total == sum(rows)
    # the cache's contents: hot rows of an earlier sample, or none, or all
    sample = _skewed_idx(rng, 4000, rows)
    if cache_rows == "none":
        chosen = np.zeros(0, np.int64)
    elif cache_rows == "all":
        chosen = rng.permutation(total).astype(np.int64)
    else:
        chosen, n = O.hot_rows(sample, rows, 300)
        chosen = chosen[:n]
    C = chosen.size
    tdt = torch.bfloat16 if dtype == eg.BF16 else torch.float32
    cache = torch.empty((max(C, 1), D_h), dtype=tdt, device="cuda")
    cmap = torch.empty(total, dtype=torch.int32, device="cuda")
    rows_d = dev(chosen) if C else torch.zeros(1, dtype=torch.int64, device="cuda")
    eg.engram_hostcache_fill(cfg, host.data_ptr(), rows_d, C, cache, cmap)
    torch.cuda.synchronize()
    # the map: slot i for chosen[i], -1 elsewhere; the cache rows exact copies
    want_map = np.full(total, -1, np.int32)
    want_map[chosen] = np.arange(C, dtype=np.int32)
    assert np.array_equal(cmap.cpu().numpy(), want_map)
    flat = np.concatenate([t.reshape(-1, D_h) for t in tb])
    if C:
        got_cache = bf16_bits(cache) if dtype == eg.BF16 else cache.cpu().numpy()
        assert np.array_equal(got_cache[:C], flat[chosen])
    # a batch from the same distribution, gathered through the cache
    N = 2500
    idx = _skewed_idx(rng, N, rows)
    e = torch.full((N, J * D_h), 3, dtype=tdt, device="cuda")
    n_miss = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    nb = eg.engram_workspace_size(cfg, eg.WS_HOSTCACHE_GATHER, N)
    side = torch.cuda.Stream()
    done = torch.cuda.Event()
    side.wait_stream(torch.cuda.current_stream())
    eg.engram_forward_hostcache(cfg, dev(idx), host.data_ptr(), cache, cmap, N, e, n_miss,
                                _ws(nb), nb, side, done)
    torch.cuda.current_stream().wait_event(done)
    want = O.gather(idx, tb)
    got = bf16_bits(e) if dtype == eg.BF16 else e.cpu().numpy()
    assert np.array_equal(got, want)
    base = np.concatenate([[0], np.cumsum(rows)[:-1]])
    valid = idx >= 0
    packed = (base[None, :] + np.where(valid, idx, 0))
    want_miss = int(np.sum(valid & (want_map[packed] < 0)))
    assert int(n_miss.item()) == want_miss
    if cache_rows == "none":
        assert want_miss == int(valid.sum())
    if cache_rows == "all":
        assert want_miss == 0
    assert eg.engram_get_status() == 0


def test_hostcache_flags_bad_rows_and_slots():
    """A cache row out of the table and a slot out of its head's range set
    ENGRAM_STATUS_BAD_INDEX; the gather still fills the valid rows."""
    rng = np.random.default_rng(9)
    K, D_h = 2, 16
    rows = synth.primes_at_most(501, 2 * K)
    tb, host = _host_table(rng, rows, D_h, eg.F32)
    cfg = eg.make_cfg(K, D_h, 256, 1, 1000, 770, eg.F32, rows, np.ones((2 * K, 3), np.uint64))
    total = eg.engram_table_rows(cfg)
    cache = torch.empty((2, D_h), device="cuda")
    cmap = torch.empty(total, dtype=torch.int32, device="cuda")
    eg.engram_hostcache_fill(cfg, host.data_ptr(), dev(np.array([3, total], np.int64)), 2, cache,
                             cmap)
    assert eg.engram_get_status() & eg.STATUS_BAD_INDEX
    idx = np.array([[0, 1, 2, 3], [5, rows[1], 0, -1]], np.int32)  # rows[1] is out of head 1
    e = torch.empty((2, 4 * D_h), device="cuda")
    nb = eg.engram_workspace_size(cfg, eg.WS_HOSTCACHE_GATHER, 2)
    eg.engram_forward_hostcache(cfg, dev(idx), host.data_ptr(), cache, cmap, 2, e, None,
                                _ws(nb), nb, None, None)
    assert eg.engram_get_status() & eg.STATUS_BAD_INDEX
    ok = np.where(idx == rows[1], -1, idx)  # the bad slot reads no row: zeros
    assert np.array_equal(e.cpu().numpy(), O.gather(ok, tb))
