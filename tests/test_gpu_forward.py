"""Parity of engram_forward with the oracle.

fp32 layers: out and alpha within 1e-5 max relative error.  bf16 layers
(tensor-core path): within 2e-2, checked at unit scale (tables N(0,1), W
N(0, 1/E)) where the Engram term is as large as h, so an error anywhere in the
gate, value, conv or residual shows in `out`; and at the 27B-shaped layer's
own scale on sampled tokens, where alpha carries the key path.
"""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O
from tests.engram_cases import (Layer, bf16_bits, bf16_dev, cfg_of, dev, gpu_hash, gpu_vocab_proj,
                                max_rel_err, packed_table, ws)

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2


def _alpha(layer, N, M):
    return layer.saved[: N * M * 4].view(torch.float32).cpu().numpy().reshape(N, M)


def _f32_case(B, T, M, d, seed, K=2, D_h=16, V=1000):
    rng = np.random.default_rng(seed)
    rows = [1009] * (2 * K)
    w = synth.custom("f32case", seed, B, T, V, K, D_h, d, "f32", rows, M=M)
    inp = synth.host_inputs(w)
    proj_ref, V_c = O.build_vocab_proj(inp["keys"])
    idx_ref = O.hash_indices(proj_ref, inp["ids"], inp["mult"], inp["rows"], K, V_c)
    e = O.gather(idx_ref.reshape(-1, w.J), inp["tables"])
    h = inp["h"].reshape(w.N, M, d)
    ref = O.layer_forward(e, h, inp["Wk"], inp["Wv"], inp["conv_w"], T)
    cfg = cfg_of(w, inp["mult"], V_c)
    proj, _ = gpu_vocab_proj(inp["keys"])
    idx = gpu_hash(cfg, proj, dev(inp["ids"]), B, T)
    L = Layer(cfg, B, T, packed_table(inp["tables"]), dev(inp["h"]), dev(inp["Wk"]),
              dev(inp["Wv"]), dev(inp["conv_w"]), torch.float32)
    out = L.forward(idx).cpu().numpy().reshape(w.N, M, d)
    return out, ref, _alpha(L, w.N, M), L, idx, inp, ref


@pytest.mark.parametrize("B,T,M", [(1, 64, 1), (1, 64, 4), (3, 37, 2), (2, 1, 1), (1, 2, 3),
                                   (4, 3, 1), (2, 129, 1)])
def test_forward_f32(B, T, M):
    out, ref, alpha, *_ = _f32_case(B, T, M, 64, seed=B * 1000 + T * 10 + M)
    assert max_rel_err(out, ref["out"]) <= TOL_F32
    assert max_rel_err(alpha, ref["alpha"]) <= TOL_F32


def test_forward_f32_zero_value_returns_h():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    cfg = cfg_of(w, inp["mult"], w.V_c)
    proj, _ = gpu_vocab_proj(inp["keys"])
    idx = gpu_hash(cfg, proj, dev(inp["ids"]), w.B, w.T)
    L = Layer(cfg, w.B, w.T, packed_table(inp["tables"]), dev(inp["h"]), dev(inp["Wk"]),
              dev(np.zeros_like(inp["Wv"])), dev(inp["conv_w"]), torch.float32)
    out = L.forward(idx).cpu().numpy()
    assert np.array_equal(out, inp["h"])


def test_forward_f32_empty():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    cfg = cfg_of(w, inp["mult"], w.V_c)
    L = Layer(cfg, 1, 1, packed_table(inp["tables"]), dev(inp["h"][:, :1]), dev(inp["Wk"]),
              dev(inp["Wv"]), dev(inp["conv_w"]), torch.float32)
    eg.engram_forward(cfg, None, L.table, L.e, L.h, L.Wk, L.Wv, L.conv_w, None, L.out, L.saved,
                      0, 64, L.fws, L.fws_bytes)


# ------------------------------------------------------------------ bf16 path

def _bf16_unit_case(B, T, d, K, D_h, seed, rows=None, decode_steps=0):
    """Unit-scale bf16 layer: returns GPU and oracle outputs."""
    rng = np.random.default_rng(seed)
    J = 2 * K
    E = J * D_h
    rows = rows or synth.primes_at_most(2003, J)
    N = B * T
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    h = rng.standard_normal((B, T, 1, d)).astype(np.float32)
    conv_w = (rng.standard_normal((d, 4)) * 0.5).astype(np.float32)
    idx = np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32)
    tb = [synth.to_bf16_bits(t) for t in tables]
    e_bits = O.gather(idx, tb)
    ref = O.layer_forward_bf16(e_bits, synth.to_bf16_bits(h).reshape(N, 1, d),
                               synth.to_bf16_bits(Wk), synth.to_bf16_bits(Wv), conv_w, T)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64))
    L = Layer(cfg, B, T, packed_table(tables, "bf16"), bf16_dev(h), bf16_dev(Wk), bf16_dev(Wv),
              dev(conv_w), torch.bfloat16)
    out = L.forward(dev(idx.reshape(B, T, J)))
    got = O.bf16_bits_to_f64(bf16_bits(out)).reshape(N, 1, d)
    assert np.array_equal(bf16_bits(L.e), e_bits)
    return got, ref, _alpha(L, N, 1)


@pytest.mark.parametrize("B,T,d,K,D_h", [
    (3, 100, 256, 2, 32),      # narrow tiles (N=64), ragged last tile
    (1, 1, 256, 2, 32),        # a single token
    (4, 2, 256, 2, 16),        # every token within the conv's start-up
    (2, 2500, 512, 2, 32),     # wide tiles (N=256), 40 overlapping V tiles of 125
    (1, 4100, 256, 4, 16),     # wide tiles with several sequences per tile boundary
])
def test_forward_bf16_unit_scale(B, T, d, K, D_h):
    got, ref, alpha = _bf16_unit_case(B, T, d, K, D_h, seed=B + T + d)
    assert max_rel_err(got, O.bf16_bits_to_f64(ref["out_bits"])) <= TOL_BF16
    assert max_rel_err(alpha, ref["alpha"]) <= TOL_BF16


def test_forward_bf16_zero_value_returns_h_exactly():
    rng = np.random.default_rng(5)
    B, T, d, K, D_h = 2, 300, 256, 2, 32
    J, E, N = 4, 128, B * T
    rows = synth.primes_at_most(2003, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    h = rng.standard_normal((B, T, 1, d)).astype(np.float32)
    idx = np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64))
    L = Layer(cfg, B, T, packed_table(tables, "bf16"), bf16_dev(h),
              bf16_dev(rng.standard_normal((1, d, E)).astype(np.float32)),
              bf16_dev(np.zeros((d, E), np.float32)), dev(np.ones((d, 4), np.float32)),
              torch.bfloat16)
    out = L.forward(dev(idx.reshape(B, T, J)))
    assert np.array_equal(bf16_bits(out), synth.to_bf16_bits(h))


def test_forward_bf16_multibranch_unsupported():
    d, K, D_h = 256, 2, 32
    cfg = eg.make_cfg(K, D_h, d, 2, 1000, 770, eg.BF16, [1009] * 4, np.ones((4, 3), np.uint64))
    t = torch.zeros(1 << 16, dtype=torch.bfloat16, device="cuda")
    w = ws(1 << 20)
    with pytest.raises(eg.EngramError) as ex:
        eg.engram_forward(cfg, t, t, t, t, t, t, t.float(), None, t, None, 1, 8, w, 1 << 20)
    assert ex.value.rc == -4


@pytest.mark.parametrize("B,d,K,D_h", [
    (300, 256, 2, 32),     # more sequences than one token tile: plain narrow tiles
    (200, 512, 2, 128),    # split units (each tile's K in two halves), ragged token tile
    (1, 256, 4, 64),       # split units, a single sequence
    (256, 256, 2, 256),    # split units, full token tiles, 8 K steps a half
    (1024, 4096, 2, 64),   # more tiles than CTA pairs fit at once: several per pair
])
def test_forward_bf16_decode_state(B, d, K, D_h):
    """One token per sequence, 6 steps, conv state carried across steps, against
    the oracle's decode step (and through it the sequence forward)."""
    rng = np.random.default_rng(44 + B + D_h)
    steps = 6
    J, E = 2 * K, 2 * K * D_h
    rows = synth.primes_at_most(3001, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    conv_w = (rng.standard_normal((d, 4)) * 0.5).astype(np.float32)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64))
    tb = [synth.to_bf16_bits(t) for t in tables]
    L = Layer(cfg, B, 1, packed_table(tables, "bf16"), None, bf16_dev(Wk), bf16_dev(Wv),
              dev(conv_w), torch.bfloat16)
    state = torch.zeros((B, 1, 3, d), dtype=torch.float32, device="cuda")
    st_ref = np.zeros((B, 1, 3, d))
    for s in range(steps):
        h = rng.standard_normal((B, 1, 1, d)).astype(np.float32)
        idx = np.stack([rng.integers(0, P, B) for P in rows], -1).astype(np.int32)
        L.h = bf16_dev(h)
        out = L.forward(dev(idx.reshape(B, 1, J)), conv_state=state)
        e_ref = O.bf16_bits_to_f64(O.gather(idx, tb))
        o_ref, a_ref, st_ref = O.decode_step(
            e_ref, O.bf16_bits_to_f64(synth.to_bf16_bits(h)).reshape(B, 1, d),
            O.bf16_bits_to_f64(synth.to_bf16_bits(Wk)), O.bf16_bits_to_f64(synth.to_bf16_bits(Wv)),
            conv_w, st_ref)
        got = O.bf16_bits_to_f64(bf16_bits(out)).reshape(B, 1, d)
        want = O.bf16_bits_to_f64(O.f64_to_bf16_bits(o_ref))
        assert max_rel_err(got, want) <= TOL_BF16, s
        assert max_rel_err(state.cpu().numpy(), st_ref) <= TOL_BF16, s
        assert max_rel_err(_alpha(L, B, 1), a_ref) <= TOL_BF16, s


def test_forward_bf16_given_e_matches_gathered():
    """table = NULL: the layer reads e as given (rows gathered elsewhere, e.g.
    from a host-resident table) and gives the same output."""
    rng = np.random.default_rng(3)
    B, T, d, K, D_h = 2, 200, 256, 2, 32
    J, E, N = 4, 128, B * T
    rows = synth.primes_at_most(2003, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    idx = dev(np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32).reshape(B, T, J))
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64))
    args = (bf16_dev(rng.standard_normal((B, T, 1, d)).astype(np.float32)),
            bf16_dev((rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)),
            bf16_dev((rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)),
            dev(rng.standard_normal((d, 4)).astype(np.float32)), torch.bfloat16)
    L1 = Layer(cfg, B, T, packed_table(tables, "bf16"), *args)
    o1 = L1.forward(idx).clone()
    L2 = Layer(cfg, B, T, None, *args)
    L2.e.copy_(L1.e)
    o2 = L2.forward(idx, table=False)
    assert torch.equal(o1, o2)


def test_forward_layer27b_sampled():
    """The 27B-shaped layer at full size (8 x 4,096 tokens, d 2,560, 16 heads x
    80 dims, 5.7B-parameter table) in the launch configuration of the timed
    step.  Sampled tokens (sequence starts, tile seams of both passes, the last
    token) against the oracle recomputed from their 4-token windows."""
    w = synth.workload("layer27b")
    ids, keys = synth.host_ids_keys(w)
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    proj_ref, V_c = O.build_vocab_proj(keys)
    idx_ref = O.hash_indices(proj_ref, ids, mult, np.array(w.rows), w.K, V_c).reshape(-1, w.J)
    table = synth.device_table(w)
    dense = synth.device_dense(w)
    cfg = cfg_of(w, mult, V_c)
    proj, _ = gpu_vocab_proj(keys)
    idx = gpu_hash(cfg, proj, dev(ids), w.B, w.T)
    L = Layer(cfg, w.B, w.T, table, dense["h"], dense["Wk"], dense["Wv"], dense["conv_w"],
              torch.bfloat16)
    out = L.forward(idx)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    alpha = _alpha(L, w.N, 1)[:, 0]
    Wk = O.bf16_bits_to_f64(bf16_bits(dense["Wk"]))
    Wv = O.bf16_bits_to_f64(bf16_bits(dense["Wv"]))
    conv_w = dense["conv_w"].cpu().numpy()
    base = np.concatenate([[0], np.cumsum(w.rows)[:-1]])
    rng = np.random.default_rng(1)
    sample = set(rng.choice(w.N, size=96, replace=False).tolist())
    # sequence starts, and the seams of both passes' tiles (pass K: 256-token
    # pair tiles; pass V: 256-token tiles advancing by 253 with a 3-token halo)
    sample |= {0, 1, 2, 3, 124, 125, 126, 127, 128, 129, 249, 250, 251, 252, 253, 254, 255, 256,
               257, 502, 503, 505, 506, 507, 4095, 4096, 4097, 4098, w.N - 1, w.N - 2,
               253 * 129, 253 * 129 - 1, 253 * 129 + 2, 253 * 129 + 3}
    errs, aerrs = [], []
    for n in sorted(sample):
        p = n % w.T
        lo = n - min(p, 3)
        win = list(range(lo, n + 1))
        e_bits = np.stack([np.concatenate([
            bf16_bits(table[(base[j] + idx_ref[m, j]) * w.D_h:(base[j] + idx_ref[m, j] + 1) * w.D_h])
            for j in range(w.J)]) for m in win])
        h_bits = np.stack([bf16_bits(dense["h"].view(w.N, w.d)[m]) for m in win])[:, None, :]
        r = O.layer_forward(O.bf16_bits_to_f64(e_bits), O.bf16_bits_to_f64(h_bits), Wk, Wv,
                            conv_w, len(win))
        want = O.bf16_bits_to_f64(O.f64_to_bf16_bits(r["out"][-1, 0]))
        got = O.bf16_bits_to_f64(bf16_bits(out.view(w.N, w.d)[n]))
        errs.append(max_rel_err(got, want))
        aerrs.append(abs(alpha[n] - r["alpha"][-1, 0]) / r["alpha"][-1, 0])
    assert max(errs) <= TOL_BF16, max(errs)
    assert max(aerrs) <= TOL_BF16, max(aerrs)
    del table, dense, L
    torch.cuda.empty_cache()


def test_decode_full_size_sampled():
    """The decode workload at full size (256 sequences x 1 token per step,
    d 4,096, 16 heads x 128 dims, 13B-parameter table) in the launch
    configuration of the timed decode step, for 4 steps.  Hash indices of
    every sequence bit-exact; out, alpha and the conv state of sampled
    sequences (both CTAs of a pair, tile seams, first and last) against the
    oracle's decode step carried across the steps."""
    w = synth.workload("decode")
    ids, keys = synth.host_ids_keys(w)
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    proj_ref, V_c = O.build_vocab_proj(keys)
    table = synth.device_table(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(41)
    Wk_d = (torch.randn((1, w.d, w.E), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    Wv_d = (torch.randn((w.d, w.E), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    cw_d = torch.randn((w.d, 4), generator=g, device="cuda") * 0.5
    cfg = cfg_of(w, mult, V_c)
    proj, _ = gpu_vocab_proj(keys)
    L = Layer(cfg, w.B, 1, table, None, Wk_d, Wv_d, cw_d, torch.bfloat16)
    state = torch.full((w.B, 2), V_c, dtype=torch.int32, device="cuda")
    conv = torch.zeros((w.B, 1, 3, w.d), dtype=torch.float32, device="cuda")
    Wk = O.bf16_bits_to_f64(bf16_bits(Wk_d))
    Wv = O.bf16_bits_to_f64(bf16_bits(Wv_d))
    conv_w = cw_d.cpu().numpy()
    base = np.concatenate([[0], np.cumsum(w.rows)[:-1]])
    sample = np.array([0, 1, 31, 32, 33, 63, 64, 65, 127, 128, 129, 191, 192, 254, 255])
    st_ref = np.full((w.B, 2), V_c, dtype=np.int32)
    conv_ref = np.zeros((len(sample), 1, 3, w.d))
    for step in range(4):
        h_d = torch.randn((w.B, 1, 1, w.d), generator=g, device="cuda").to(torch.bfloat16)
        L.h = h_d
        idx = gpu_hash(cfg, proj, dev(ids[step].copy()), w.B, 1, state=state)
        out = L.forward(idx, conv_state=conv)
        torch.cuda.synchronize()
        assert eg.engram_get_status() == 0
        idx_ref, st_ref = O.hash_indices_decode(proj_ref, ids[step], st_ref, mult,
                                                np.array(w.rows), w.K)
        assert np.array_equal(idx.cpu().numpy().reshape(w.B, w.J), idx_ref), step
        e_bits = np.stack([np.concatenate([
            bf16_bits(table[(base[j] + idx_ref[b, j]) * w.D_h:(base[j] + idx_ref[b, j] + 1) * w.D_h])
            for j in range(w.J)]) for b in sample])
        h_bits = bf16_bits(h_d.view(w.B, w.d)[torch.from_numpy(sample).cuda()])
        o_ref, a_ref, conv_ref = O.decode_step(
            O.bf16_bits_to_f64(e_bits), O.bf16_bits_to_f64(h_bits)[:, None, :], Wk, Wv, conv_w,
            conv_ref)
        got = O.bf16_bits_to_f64(bf16_bits(out.view(w.B, w.d)))[sample]
        want = O.bf16_bits_to_f64(O.f64_to_bf16_bits(o_ref[:, 0]))
        assert max_rel_err(got, want) <= TOL_BF16, step
        assert max_rel_err(_alpha(L, w.B, 1)[sample], a_ref) <= TOL_BF16, step
        assert max_rel_err(conv.cpu().numpy()[sample], conv_ref) <= TOL_BF16, step
    del table, L
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,T,d,dtype", [
    (3, 100, 256, "bf16"),    # narrow tensor-core tiles
    (2, 2500, 512, "bf16"),   # wide tiles: pass V overwrites h while later tiles still load it
    (2, 37, 64, "f32"),       # CUDA-core path
])
def test_forward_in_place_equals_separate_output(B, T, d, dtype):
    """out == h (the residual applied in place) gives bit for bit the output of
    a run with a separate out buffer."""
    rng = np.random.default_rng(B * 7 + T)
    K, D_h = 2, 32 if dtype == "bf16" else 16
    J, E, N = 2 * K, 2 * K * D_h, B * T
    rows = synth.primes_at_most(2003, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    h = rng.standard_normal((B, T, 1, d)).astype(np.float32)
    conv_w = (rng.standard_normal((d, 4)) * 0.5).astype(np.float32)
    idx = dev(np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32).reshape(B, T, J))
    t_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
    put = bf16_dev if dtype == "bf16" else dev
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16 if dtype == "bf16" else eg.F32, rows,
                      np.ones((J, 3), np.uint64))
    L = Layer(cfg, B, T, packed_table(tables, dtype), put(h), put(Wk), put(Wv), dev(conv_w),
              t_dtype)
    sep = L.forward(idx).clone()
    alpha_sep = _alpha(L, N, 1).copy()
    L.out = L.h                     # out aliases h
    L.forward(idx)
    torch.cuda.synchronize()
    assert torch.equal(L.h, sep)
    assert np.array_equal(_alpha(L, N, 1), alpha_sep)
    assert eg.engram_get_status() == 0


@pytest.mark.parametrize("dtype,B,d,K,D_h,flags", [
    ("bf16", 37, 256, 2, 32, 0),                  # narrow tensor-core tiles, ragged batch
    ("bf16", 300, 512, 4, 16, eg.CONV_DILATED),   # two token tiles, dilated conv state
    ("bf16", 100, 512, 4, 64, 0),                 # split units (K in two halves per tile)
    ("bf16", 256, 256, 2, 128, eg.CONV_DILATED),  # split units, dilated conv state
    ("bf16", 700, 2048, 2, 64, eg.CONV_DILATED),  # several tiles per CTA pair, dilated
    ("f32", 5, 64, 2, 16, 0),                     # fp32 layer
    ("f32", 9, 64, 3, 16, 0),                     # J = 6 heads (two per hash thread)
])
def test_decode_step_equals_hash_then_forward(dtype, B, d, K, D_h, flags):
    """engram_decode_step (hash and gather in one kernel, then the layer) gives
    the same bits as engram_hash_indices followed by engram_forward, step after
    step: slots, n-gram state, gathered rows, output and conv state."""
    rng = np.random.default_rng(B * 7 + d)
    J, E = 2 * K, 2 * K * D_h
    rows = synth.primes_at_most(3001, J)
    V = 1000
    keys = synth.merge_keys(np.random.default_rng(5), V, synth.compressed_vocab(V))
    proj, V_c = gpu_vocab_proj(keys)
    mult = synth.hash_multipliers(77, J)
    cfg = eg.make_cfg(K, D_h, d, 1, V, V_c, eg.BF16 if dtype == "bf16" else eg.F32, rows, mult,
                      flags=flags)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    to = (lambda x: bf16_dev(x)) if dtype == "bf16" else (lambda x: dev(x))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    table = packed_table(tables, dtype)
    Wk = to((rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32))
    Wv = to((rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32))
    cw = dev((rng.standard_normal((d, 4)) * 0.5).astype(np.float32))
    dil = 3 if flags & eg.CONV_DILATED else 1
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, B)
    paths = []
    for _ in range(2):
        paths.append(dict(
            state=torch.full((B, 2), V_c, dtype=torch.int32, device="cuda"),
            conv=torch.zeros((B, 1, 3 * dil, d), dtype=torch.float32, device="cuda"),
            idx=torch.empty((B, 1, J), dtype=torch.int32, device="cuda"),
            e=torch.empty((B, E), dtype=tdt, device="cuda"),
            out=torch.empty((B, 1, 1, d), dtype=tdt, device="cuda"),
            ws=ws(fb)))
    a, b = paths
    for step in range(6):
        ids = dev(rng.integers(0, V, size=B).astype(np.int32))
        h = to(rng.standard_normal((B, 1, 1, d)).astype(np.float32))
        eg.engram_hash_indices(cfg, proj, ids, B, 1, a["state"], a["idx"])
        eg.engram_forward(cfg, a["idx"], table, a["e"], h, Wk, Wv, cw, a["conv"], a["out"], None,
                          B, 1, a["ws"], fb)
        eg.engram_decode_step(cfg, proj, ids, b["state"], b["idx"], table, b["e"], h, Wk, Wv, cw,
                              b["conv"], b["out"], B, b["ws"], fb)
        torch.cuda.synchronize()
        assert eg.engram_get_status() == 0
        for name in ("idx", "state", "e", "out", "conv"):
            assert torch.equal(a[name], b[name]), (step, name)


def test_decode_steps_on_two_streams_at_once():
    """Two independent decode streams (own n-gram state, conv state, buffers
    and workspace) issued on two CUDA streams with no synchronisation between
    them give the same bits as each run alone.  Each step's layer kernel
    needs all of its CTAs resident at once (its CTAs wait for one another at
    the gate); two such grids do not fit the GPU together, so this checks
    that one cannot hold part of the SMs while the other waits."""
    rng = np.random.default_rng(808)
    B, d, K, D_h = 256, 4096, 2, 64
    J, E = 2 * K, 2 * K * D_h
    rows = synth.primes_at_most(3001, J)
    V = 1000
    keys = synth.merge_keys(np.random.default_rng(6), V, synth.compressed_vocab(V))
    proj, V_c = gpu_vocab_proj(keys)
    cfg = eg.make_cfg(K, D_h, d, 1, V, V_c, eg.BF16, rows, synth.hash_multipliers(78, J))
    table = packed_table([rng.standard_normal((P, D_h)).astype(np.float32) for P in rows], "bf16")
    Wk = bf16_dev((rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32))
    Wv = bf16_dev((rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32))
    cw = dev((rng.standard_normal((d, 4)) * 0.5).astype(np.float32))
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, B)
    steps = 6
    inputs = [[(dev(rng.integers(0, V, size=B).astype(np.int32)),
                bf16_dev(rng.standard_normal((B, 1, 1, d)).astype(np.float32)))
               for _ in range(steps)] for _ in range(2)]

    def fresh():
        return dict(state=torch.full((B, 2), V_c, dtype=torch.int32, device="cuda"),
                    conv=torch.zeros((B, 1, 3, d), dtype=torch.float32, device="cuda"),
                    e=torch.empty((B, E), dtype=torch.bfloat16, device="cuda"),
                    out=torch.empty((B, steps, d), dtype=torch.bfloat16, device="cuda"),
                    ws=ws(fb))

    def step(p, k, ids, h, stream):
        with torch.cuda.stream(stream):  # o belongs to the stream that uses it
            o = torch.empty((B, 1, 1, d), dtype=torch.bfloat16, device="cuda")
            eg.engram_decode_step(cfg, proj, ids, p["state"], None, table, p["e"], h, Wk, Wv, cw,
                                  p["conv"], o, B, p["ws"], fb, stream)
            p["out"][:, k] = o[:, 0, 0]

    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    alone = [fresh(), fresh()]
    torch.cuda.synchronize()
    for i in range(2):
        for k in range(steps):
            step(alone[i], k, *inputs[i][k], s1)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    both = [fresh(), fresh()]
    torch.cuda.synchronize()
    for k in range(steps):
        step(both[0], k, *inputs[0][k], s1)
        step(both[1], k, *inputs[1][k], s2)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    for i in range(2):
        for name in ("state", "conv", "out"):
            assert torch.equal(both[i][name], alone[i][name]), (i, name)
