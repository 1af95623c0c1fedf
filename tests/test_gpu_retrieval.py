"""Parity of the retrieval kernels (vocabulary projection, fused
compress + n-gram + hash, gather) with the oracle: bit-exact."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O
from tests.engram_cases import (bf16_bits, bf16_dev, cfg_of, dev, gpu_hash, gpu_vocab_proj,
                                packed_table)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "layer27b"])
def test_vocab_proj_bit_exact(name):
    w = synth.workload(name)
    _, keys = synth.host_ids_keys(w) if name != "tiny" else (None, synth.host_inputs(w)["keys"])
    want, vc_want = O.build_vocab_proj(keys)
    proj, V_c = gpu_vocab_proj(keys)
    assert V_c == vc_want == w.V_c
    assert np.array_equal(proj.cpu().numpy(), want)


def test_vocab_proj_small_vocabularies():
    rng = np.random.default_rng(0)
    for V in [1, 2, 5, 31, 2047, 2048, 2049, 5000]:
        keys = rng.integers(0, max(V // 3, 1), size=V).astype(np.int64) * 7919 - 3
        want, vc = O.build_vocab_proj(keys)
        proj, V_c = gpu_vocab_proj(keys)
        assert V_c == vc
        assert np.array_equal(proj.cpu().numpy(), want)


def _hash_case(w, ids, B, T):
    inp_keys = synth.host_inputs(w)["keys"] if w.V == 1000 else synth.host_ids_keys(w)[1]
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    proj_ref, V_c = O.build_vocab_proj(inp_keys)
    want = O.hash_indices(proj_ref, ids, mult, np.array(w.rows), w.K, V_c)
    proj, _ = gpu_vocab_proj(inp_keys)
    cfg = cfg_of(w, mult, V_c)
    got = gpu_hash(cfg, proj, dev(ids.astype(np.int32)), B, T)
    return got.cpu().numpy(), want


@pytest.mark.parametrize("name", ["tiny", "layer27b"])
def test_hash_bit_exact(name):
    w = synth.workload(name)
    ids = synth.host_ids_keys(w)[0] if name != "tiny" else synth.host_inputs(w)["ids"]
    got, want = _hash_case(w, ids, w.B, w.T)
    assert np.array_equal(got, want)
    assert eg.engram_get_status() == 0


@pytest.mark.parametrize("B,T", [(3, 37), (5, 1), (4, 2), (2, 3), (1, 257), (7, 33)])
def test_hash_ragged_shapes(B, T):
    w = synth.workload("tiny")
    ids = np.random.default_rng(B * 100 + T).integers(0, w.V, size=(B, T)).astype(np.int32)
    got, want = _hash_case(w, ids, B, T)
    assert np.array_equal(got, want)


def test_hash_empty_batch():
    w = synth.workload("tiny")
    mult = synth.hash_multipliers(1, w.J)
    cfg = cfg_of(w, mult, w.V_c)
    proj = torch.zeros(w.V, dtype=torch.int32, device="cuda")
    ids = torch.zeros(16, dtype=torch.int32, device="cuda")
    idx = torch.full((16,), 7, dtype=torch.int32, device="cuda")
    eg.engram_hash_indices(cfg, proj, ids, 0, 5, None, idx)
    torch.cuda.synchronize()
    assert (idx == 7).all()


def test_hash_decode_state_bit_exact():
    """All 2,000 decode steps of the decode workload (256 sequences): the
    indices of every step and the rolling n-gram state bit-exact."""
    w = synth.workload("decode")
    ids, keys = synth.host_ids_keys(w)          # [steps, B]
    steps = w.steps
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    proj_ref, V_c = O.build_vocab_proj(keys)
    proj, _ = gpu_vocab_proj(keys)
    cfg = cfg_of(w, mult, V_c)
    state = dev(np.full((w.B, 2), V_c, dtype=np.int32))
    ids_d = dev(ids)
    idx_all = torch.empty((steps, w.B, 1, w.J), dtype=torch.int32, device="cuda")
    mid_state = None
    for s in range(steps):
        eg.engram_hash_indices(cfg, proj, ids_d[s], w.B, 1, state, idx_all[s])
        if s == steps // 2:
            mid_state = state.cpu().numpy()
    got = idx_all.cpu().numpy()[:, :, 0]
    state_ref = np.full((w.B, 2), V_c, dtype=np.int32)
    for s in range(steps):
        want, state_ref = O.hash_indices_decode(proj_ref, ids[s], state_ref, mult,
                                                np.array(w.rows), w.K)
        assert np.array_equal(got[s], want), s
        if s == steps // 2:
            assert np.array_equal(mid_state, state_ref)
    assert np.array_equal(state.cpu().numpy(), state_ref)


def test_hash_bad_ids_flag_and_minus_one():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    ids = inp["ids"].copy()
    ids[0, 10] = -5
    ids[0, 40] = w.V
    mult = inp["mult"]
    proj, V_c = gpu_vocab_proj(inp["keys"])
    cfg = cfg_of(w, mult, V_c)
    eg.engram_get_status()
    got = gpu_hash(cfg, proj, dev(ids), w.B, w.T).cpu().numpy()[0]
    assert eg.engram_get_status() & eg.STATUS_BAD_ID
    K = w.K
    for t in (10, 40):
        assert (got[t] == -1).all()
        assert (got[t + 1] == -1).all()                  # both orders see c_t
        assert (got[t + 2, K:] == -1).all() and (got[t + 2, :K] >= 0).all()
    # tokens whose n-grams avoid the bad ids agree with the oracle on clean ids
    clean = inp["ids"].copy()
    proj_ref, _ = O.build_vocab_proj(inp["keys"])
    want = O.hash_indices(proj_ref, clean, mult, inp["rows"], K, V_c)[0]
    ok = np.ones(w.T, bool)
    ok[[10, 11, 12, 40, 41, 42]] = False
    assert np.array_equal(got[ok], want[ok])
    assert eg.engram_get_status() == 0


def test_gather_fp32_bit_exact():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    proj_ref, V_c = O.build_vocab_proj(inp["keys"])
    idx = O.hash_indices(proj_ref, inp["ids"], inp["mult"], inp["rows"], w.K, V_c)
    want = O.gather(idx.reshape(-1, w.J), inp["tables"])
    cfg = cfg_of(w, inp["mult"], V_c)
    e = torch.empty((w.N, w.E), dtype=torch.float32, device="cuda")
    eg.engram_gather(cfg, dev(idx), packed_table(inp["tables"]), w.N, e)
    assert np.array_equal(e.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_gather_bf16_bit_exact_ragged():
    # bf16 rows of 80 (160 bytes = 10 vectors), several thousand tokens with a
    # ragged tail, random slots over small prime tables
    rng = np.random.default_rng(9)
    K, D_h = 8, 80
    rows = synth.primes_at_most(5003, 16)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    N = 3001
    idx = np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32)
    tb = [synth.to_bf16_bits(t) for t in tables]
    want = O.gather(idx, tb)                               # bf16 bit patterns
    cfg = eg.make_cfg(K, D_h, 256, 1, 1000, 770, eg.BF16, rows, np.ones((16, 3), np.uint64))
    e = torch.empty((N, 16 * D_h), dtype=torch.bfloat16, device="cuda")
    eg.engram_gather(cfg, dev(idx), packed_table(tables, "bf16"), N, e)
    assert np.array_equal(bf16_bits(e), want)


def test_gather_out_of_range_index_gives_zero_row_and_flag():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    cfg = cfg_of(w, inp["mult"], w.V_c)
    idx = np.zeros((4, w.J), np.int32)
    idx[1, 2] = 1009          # one past the end of head 2
    idx[2, 0] = -1            # an invalid slot from the hash: zeros, no new flag
    e = torch.full((4, w.E), 5.0, dtype=torch.float32, device="cuda")
    eg.engram_get_status()
    eg.engram_gather(cfg, dev(idx), packed_table(inp["tables"]), 4, e)
    st = eg.engram_get_status()
    got = e.cpu().numpy()
    assert st & eg.STATUS_BAD_INDEX
    assert not got[1, 2 * w.D_h:3 * w.D_h].any()
    assert not got[2, 0:w.D_h].any()
    want = O.gather(np.zeros((1, w.J), np.int32), inp["tables"])[0]
    assert np.array_equal(got[0], want)


def test_gather_full_size_sampled():
    """The 27B-shaped table (5.7B bf16 parameters, 11.4 GB) on the device and
    all 32,768 tokens gathered as in the timed step; sampled tokens checked
    bit for bit against the oracle's gather of the same rows."""
    w = synth.workload("layer27b")
    ids, keys = synth.host_ids_keys(w)
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    proj_ref, V_c = O.build_vocab_proj(keys)
    idx_ref = O.hash_indices(proj_ref, ids, mult, np.array(w.rows), w.K, V_c).reshape(-1, w.J)
    table = synth.device_table(w)
    proj, _ = gpu_vocab_proj(keys)
    cfg = cfg_of(w, mult, V_c)
    idx = gpu_hash(cfg, proj, dev(ids), w.B, w.T)
    e = torch.empty((w.N, w.E), dtype=torch.bfloat16, device="cuda")
    eg.engram_gather(cfg, idx, table, w.N, e)
    sample = np.random.default_rng(2).choice(w.N, size=512, replace=False)
    sample[:3] = [0, w.T, w.N - 1]
    base = np.concatenate([[0], np.cumsum(w.rows)[:-1]])
    for n in sample.tolist():
        rows_bits = []
        for j in range(w.J):
            r = int(base[j] + idx_ref[n, j])
            rows_bits.append(bf16_bits(table[r * w.D_h:(r + 1) * w.D_h]))
        want = O.gather(np.arange(w.J)[None, :] * 0, [rb[None, :] for rb in rows_bits])[0]
        assert np.array_equal(bf16_bits(e[n]), want), n
    del table
    torch.cuda.empty_cache()


@pytest.mark.parametrize("K", list(range(1, 17)))
def test_hash_head_counts(K):
    """Every head count the configuration allows (J = 2K up to 32: four heads
    per thread when J is a multiple of 4, else two), on a ragged batch."""
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    proj_ref, V_c = O.build_vocab_proj(inp["keys"])
    B, T = 3, 45
    ids = np.random.default_rng(K).integers(0, w.V, size=(B, T)).astype(np.int32)
    mult = synth.hash_multipliers(100 + K, 2 * K)
    rows = np.array(synth.primes_at_most(10007, 2 * K), dtype=np.int64)
    want = O.hash_indices(proj_ref, ids, mult, rows, K, V_c)
    proj, _ = gpu_vocab_proj(inp["keys"])
    cfg = eg.make_cfg(K, 16, 64, 1, w.V, V_c, eg.F32, rows, mult)
    got = gpu_hash(cfg, proj, dev(ids), B, T)
    assert np.array_equal(got.cpu().numpy(), want)


def test_gather_from_host_table_bit_exact():
    """Rows gathered over PCIe from a pinned, mapped host table on a side
    stream; the compute stream waits on the returned event."""
    rng = np.random.default_rng(21)
    K, D_h = 8, 160
    rows = synth.primes_at_most(3001, 16)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    N = 2051
    idx = np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32)
    tb = [synth.to_bf16_bits(t) for t in tables]
    want = O.gather(idx, tb)
    flat = np.concatenate([t.reshape(-1) for t in tb]).view(np.int16)
    host = torch.from_numpy(flat).pin_memory()       # page-locked, mapped into the GPU's space
    cfg = eg.make_cfg(K, D_h, 256, 1, 1000, 770, eg.BF16, rows, np.ones((16, 3), np.uint64))
    e = torch.empty((N, 16 * D_h), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    done = torch.cuda.Event()
    idx_d = dev(idx)
    side.wait_stream(torch.cuda.current_stream())
    eg.engram_forward_hosttable(cfg, idx_d, host.data_ptr(), N, e, side, done)
    torch.cuda.current_stream().wait_event(done)
    assert np.array_equal(bf16_bits(e), want)
    assert eg.engram_get_status() == 0


@pytest.mark.parametrize("N,span", [
    (2051, 5),      # every head's slots from a handful of rows: most items repeat
    (1, 3),         # a single token
    (777, 400),     # some repeats, ragged last warp
])
def test_host_table_repeats_and_invalid_slots(N, span):
    """The host gather against the oracle when rows repeat across tokens and
    heads, with -1 slots (zero rows, no status) mixed in; out-of-range slots
    give zero rows and ENGRAM_STATUS_BAD_INDEX."""
    rng = np.random.default_rng(N + span)
    K, D_h = 4, 32
    J = 2 * K
    rows = synth.primes_at_most(1009, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    idx = np.stack([rng.integers(0, span, N) for _ in rows], -1).astype(np.int32)
    idx[rng.random(idx.shape) < 0.05] = -1
    tb = [synth.to_bf16_bits(t) for t in tables]
    flat = np.concatenate([t.reshape(-1) for t in tb]).view(np.int16)
    host = torch.from_numpy(flat).pin_memory()
    cfg = eg.make_cfg(K, D_h, 256, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64))
    e = torch.full((N, J * D_h), 7.0, dtype=torch.bfloat16, device="cuda")
    eg.engram_forward_hosttable(cfg, dev(idx), host.data_ptr(), N, e)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(e), O.gather(idx, tb))
    assert eg.engram_get_status() == 0
    bad = idx.copy()
    bad[0, 0] = rows[0]
    bad[-1, J - 1] = rows[J - 1] + 5
    eg.engram_forward_hosttable(cfg, dev(bad), host.data_ptr(), N, e)
    torch.cuda.synchronize()
    assert eg.engram_get_status() & eg.STATUS_BAD_INDEX
    ref = bad.copy()
    ref[0, 0] = -1
    ref[-1, J - 1] = -1
    assert np.array_equal(bf16_bits(e), O.gather(ref, tb))


def test_gather_from_host_table_rejects_unmapped_memory():
    cfg = eg.make_cfg(8, 160, 256, 1, 1000, 770, eg.BF16, synth.primes_at_most(3001, 16),
                      np.ones((16, 3), np.uint64))
    plain = np.zeros(1 << 20, dtype=np.int16)          # ordinary pageable host memory
    idx = dev(np.zeros((4, 16), np.int32))
    e = torch.empty((4, 16 * 160), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eg.EngramError) as ex:
        eg.engram_forward_hosttable(cfg, idx, plain.ctypes.data, 4, e, None, None)
    assert ex.value.rc == -1
