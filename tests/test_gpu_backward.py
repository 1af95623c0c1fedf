"""Parity of engram_backward and engram_table_grad with the oracle.

Dense gradients (fp32 layers) within 1e-5 max relative error.  The sparse
table gradient: on the same seeded de, keys, count and row sums are
bit-identical to the oracle's ascending-token fp32 reduction; end to end
(de from the GPU's own backward) the rows agree within 1e-5.
"""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O
from tests.engram_cases import (Layer, cfg_of, dev, gpu_hash, gpu_vocab_proj, max_rel_err,
                                packed_table, ws)

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _layer(w, layer, h_dev=None):
    inp = synth.host_inputs(w, layer=layer)
    proj_ref, V_c = O.build_vocab_proj(inp["keys"])
    idx_ref = O.hash_indices(proj_ref, inp["ids"], inp["mult"], inp["rows"], w.K, V_c)
    cfg = cfg_of(w, inp["mult"], V_c)
    proj, _ = gpu_vocab_proj(inp["keys"])
    idx = gpu_hash(cfg, proj, dev(inp["ids"]), w.B, w.T)
    L = Layer(cfg, w.B, w.T, packed_table(inp["tables"]),
              dev(inp["h"]) if h_dev is None else h_dev, dev(inp["Wk"]), dev(inp["Wv"]),
              dev(inp["conv_w"]), torch.float32)
    e_ref = O.gather(idx_ref.reshape(-1, w.J), [t.astype(np.float64) for t in inp["tables"]])
    return inp, idx_ref, idx, L, e_ref


def _check_grads(g, ref, L, idx_ref, w):
    assert max_rel_err(g["dh"].cpu().numpy(), ref["dh"]) <= TOL
    assert max_rel_err(g["dWk"].cpu().numpy(), ref["dWk"]) <= TOL
    assert max_rel_err(g["dWv"].cpu().numpy(), ref["dWv"]) <= TOL
    assert max_rel_err(g["dconv_w"].cpu().numpy(), ref["dconv_w"]) <= TOL
    assert max_rel_err(g["de"].cpu().numpy(), ref["de"]) <= TOL
    # sparse table gradient: the same rows (bit-exact keys) and, since both
    # sides sum de in fp32 in ascending token order, values within TOL of the
    # oracle's reduction applied to the oracle's de
    keys_ref, rows_ref = O.table_grad_segments_fast(idx_ref, ref["de"].astype(np.float32), w.rows,
                                                    w.D_h)
    U = int(g["n_unique"].item())
    assert U == keys_ref.size
    assert np.array_equal(g["keys"][:U].cpu().numpy(), keys_ref)
    assert max_rel_err(g["rows"][:U].cpu().numpy(), rows_ref) <= TOL


@pytest.mark.parametrize("M", [1, 4])
def test_backward_single_layer(M):
    w = synth.workload("tiny") if M == 1 else synth.workload("train")
    inp, idx_ref, idx, L, e_ref = _layer(w, 0)
    L.forward(idx)
    dout = inp["dout"]
    g = L.backward(idx, dev(dout))
    ref = O.layer_backward(e_ref, inp["h"].reshape(w.N, w.M, w.d), inp["Wk"], inp["Wv"],
                           inp["conv_w"], w.T, dout.reshape(w.N, w.M, w.d))
    _check_grads(g, ref, L, idx_ref.reshape(-1, w.J), w)


def test_backward_two_layer_chain():
    """Training step of the two-layer, 4-branch workload: Engram at layers 2
    and 6, the output of layer 2 feeding layer 6; the backward of layer 6
    hands dh to layer 2 as its output gradient."""
    w = synth.workload("train")
    inp2, idx2_ref, idx2, L2, e2 = _layer(w, 2)
    L2.forward(idx2)
    inp6, idx6_ref, idx6, L6, e6 = _layer(w, 6, h_dev=L2.out)
    L6.forward(idx6)
    dout = inp2["dout"]
    g6 = L6.backward(idx6, dev(dout))
    g2 = L2.backward(idx2, g6["dh"].view(w.B, w.T, w.M, w.d))
    h0 = inp2["h"].reshape(w.N, w.M, w.d)
    f2 = O.layer_forward(e2, h0, inp2["Wk"], inp2["Wv"], inp2["conv_w"], w.T)
    assert max_rel_err(L2.out.cpu().numpy().reshape(w.N, w.M, w.d), f2["out"]) <= TOL
    # the tensors passed between the layers (out of layer 2, dh of layer 6)
    # are fp32 in this configuration: the oracle's chain stores them so too
    h6 = f2["out"].astype(np.float32).astype(np.float64)
    f6 = O.layer_forward(e6, h6, inp6["Wk"], inp6["Wv"], inp6["conv_w"], w.T)
    assert max_rel_err(L6.out.cpu().numpy().reshape(w.N, w.M, w.d), f6["out"]) <= TOL
    r6 = O.layer_backward(e6, h6, inp6["Wk"], inp6["Wv"], inp6["conv_w"], w.T,
                          dout.reshape(w.N, w.M, w.d))
    r2 = O.layer_backward(e2, h0, inp2["Wk"], inp2["Wv"], inp2["conv_w"], w.T,
                          r6["dh"].astype(np.float32).astype(np.float64))
    _check_grads(g6, r6, L6, idx6_ref.reshape(-1, w.J), w)
    _check_grads(g2, r2, L2, idx2_ref.reshape(-1, w.J), w)


def _table_grad(cfg, idx_np, de_np):
    n_tok = idx_np.shape[0]
    n = max(n_tok * cfg.J, 1)
    keys = torch.empty(n, dtype=torch.int64, device="cuda")
    rows = torch.empty((n, cfg.D_h), dtype=torch.float32, device="cuda")
    nu = torch.zeros(1, dtype=torch.int32, device="cuda")
    nb = eg.engram_workspace_size(cfg, eg.WS_TABLE_GRAD, n_tok)
    eg.engram_table_grad(cfg, dev(idx_np) if n_tok else None, dev(de_np) if n_tok else None,
                         n_tok, keys, rows, nu, ws(nb), nb)
    U = int(nu.item())
    return keys[:U].cpu().numpy(), rows[:U].cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "layer27b"])
def test_table_grad_bit_exact(name):
    w = synth.workload(name)
    if name == "tiny":
        inp = synth.host_inputs(w)
        ids, keys_v, mult = inp["ids"], inp["keys"], inp["mult"]
    else:
        ids, keys_v = synth.host_ids_keys(w)
        mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    proj_ref, V_c = O.build_vocab_proj(keys_v)
    idx = O.hash_indices(proj_ref, ids, mult, np.array(w.rows), w.K, V_c).reshape(-1, w.J)
    de = synth.seeded_floats(w.seed + 500, (w.N, w.E))
    cfg = cfg_of(w, mult, V_c)
    cfg.dtype = eg.F32
    k_ref, r_ref = O.table_grad_segments_fast(idx, de, w.rows, w.D_h)
    k, r = _table_grad(cfg, idx, de)
    assert np.array_equal(k, k_ref)
    assert np.array_equal(r.view(np.uint32), r_ref.view(np.uint32))


def test_table_grad_order_sensitive_and_invalid_slots():
    # values whose fp32 sum depends on the order: only ascending token order
    # reproduces the oracle; slots of -1 are left out
    cfg = eg.make_cfg(2, 4, 64, 1, 1000, 770, eg.F32, [7, 11, 13, 17], np.ones((4, 3), np.uint64))
    rng = np.random.default_rng(12)
    N = 5000
    idx = np.stack([rng.integers(0, P, N) for P in [7, 11, 13, 17]], -1).astype(np.int32)
    idx[rng.random((N, 4)) < 0.05] = -1
    de = (rng.standard_normal((N, 16)) * np.float32(1e6) ** rng.integers(0, 2, (N, 16))).astype(np.float32)
    k_ref, r_ref = O.table_grad_segments_fast(np.where(idx < 0, 0, idx), de, [7, 11, 13, 17], 4)
    # drop invalid items from the reference by recomputing without them
    keep = idx >= 0
    sums = {}
    base = [0, 7, 18, 31]
    for t in range(N):
        for j in range(4):
            if keep[t, j]:
                key = base[j] + int(idx[t, j])
                sums[key] = (sums.get(key, np.zeros(4, np.float32)) + de[t, 4 * j:4 * j + 4]).astype(np.float32)
    kk = np.array(sorted(sums), np.int64)
    rr = np.stack([sums[x] for x in kk.tolist()])
    k, r = _table_grad(cfg, idx, de)
    assert np.array_equal(k, kk)
    assert np.array_equal(r.view(np.uint32), rr.view(np.uint32))


def test_table_grad_empty():
    cfg = eg.make_cfg(2, 4, 64, 1, 1000, 770, eg.F32, [7, 11, 13, 17], np.ones((4, 3), np.uint64))
    k, r = _table_grad(cfg, np.zeros((0, 4), np.int32), np.zeros((0, 16), np.float32))
    assert k.size == 0 and r.size == 0
    idx = np.full((3, 4), -1, np.int32)
    k, r = _table_grad(cfg, idx, np.ones((3, 16), np.float32))
    assert k.size == 0


def test_backward_is_deterministic():
    w = synth.workload("train")
    inp, idx_ref, idx, L, _ = _layer(w, 0)
    L.forward(idx)
    g1 = L.backward(idx, dev(inp["dout"]))
    g2 = L.backward(idx, dev(inp["dout"]))
    U = int(g1["n_unique"].item())
    assert U == int(g2["n_unique"].item())
    for k in ("dh", "dWk", "dWv", "dconv_w", "de"):
        assert torch.equal(g1[k], g2[k]), k
    assert torch.equal(g1["keys"][:U], g2["keys"][:U])
    assert torch.equal(g1["rows"][:U], g2["rows"][:U])


# ---------------------------------------------------------------- bf16 layers

TOL_BF16 = 2e-2


def _bf16_backward_case(B, T, d, K, D_h, seed, flags=0, with_layer=False):
    """A unit-scale bf16 layer (tables N(0,1), W N(0,1/E)): GPU forward then
    backward, and the oracle's fp64 backward on the same bf16 values.  flags
    = eg.SAVE_KV has the forward keep k and v for the backward."""
    from tests.engram_cases import bf16_bits, bf16_dev
    rng = np.random.default_rng(seed)
    J, E, N = 2 * K, 2 * K * D_h, B * T
    rows = synth.primes_at_most(2003, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    h = rng.standard_normal((B, T, 1, d)).astype(np.float32)
    conv_w = (rng.standard_normal((d, 4)) * 0.5).astype(np.float32)
    dout = rng.standard_normal((N, 1, d)).astype(np.float32)
    idx = np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64),
                      flags=flags)
    block = conv_w.reshape(-1)
    n_scales = eg.engram_param_floats(cfg) - 4 * d
    if n_scales:  # learnable g_h, g_k (and g_v) after the conv weights
        block = np.r_[block, 1.0 + 0.3 * rng.standard_normal(n_scales)].astype(np.float32)
    L = Layer(cfg, B, T, packed_table(tables, "bf16"), bf16_dev(h), bf16_dev(Wk), bf16_dev(Wv),
              dev(block), torch.bfloat16)
    idx_d = dev(idx.reshape(B, T, J))
    L.forward(idx_d)
    g = L.backward(idx_d, dev(dout))
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    f64 = O.bf16_bits_to_f64
    e_ref = f64(O.gather(idx, [synth.to_bf16_bits(t) for t in tables]))
    assert np.array_equal(bf16_bits(L.e), O.gather(idx, [synth.to_bf16_bits(t) for t in tables]))
    vflags = ((O.NORM_SCALES if flags & eg.NORM_SCALES else 0) |
              (O.CONV_DILATED if flags & eg.CONV_DILATED else 0) |
              (O.CONV_PRENORM if flags & eg.CONV_PRENORM else 0))
    if vflags:
        ref = O.layer_backward_v(e_ref, f64(synth.to_bf16_bits(h)).reshape(N, 1, d),
                                 f64(synth.to_bf16_bits(Wk)), f64(synth.to_bf16_bits(Wv)), block,
                                 T, dout, vflags)
        ref["dconv_w"] = ref["dblock"]
    else:
        ref = O.layer_backward(e_ref, f64(synth.to_bf16_bits(h)).reshape(N, 1, d),
                               f64(synth.to_bf16_bits(Wk)), f64(synth.to_bf16_bits(Wv)), conv_w,
                               T, dout)
    ref["e"] = e_ref
    ref["Wk_bf"] = f64(synth.to_bf16_bits(Wk))
    ref["Wv_bf"] = f64(synth.to_bf16_bits(Wv))
    if with_layer:
        return g, ref, idx, rows, D_h, L
    return g, ref, idx, rows, D_h


# The gradients that leave the elementwise kernels (dh, dconv_w) are held to
# the bf16 forward's metric.  dW_k, dW_v and de come out of GEMMs whose
# operands dk and dv are rounded to bf16 once (relative error <= 2^-9 each)
# and accumulated in fp32: an element's error is then bounded by 2^-9 times
# the sum of the absolute products that form it, not by its own size (which
# cancellation can make arbitrarily small).  Each element is checked against
# twice that bound, computed from the oracle's own dk and dv.
GEMM_REL = 2.0 ** -8


def _within_gemm_bound(got, want, bound):
    excess = np.abs(got - want) - (GEMM_REL * bound + 1e-6 * np.abs(want).max())
    return float(excess.max()) <= 0.0


@pytest.mark.parametrize("B,T,d,K,D_h", [
    (3, 100, 256, 2, 32),     # narrow forward tiles, sequences of 100
    (2, 2500, 512, 2, 32),    # wide forward tiles
    (64, 1, 256, 2, 32),      # one-token sequences: every token starts and ends one
    (50, 3, 256, 2, 32),      # sequences shorter than the conv
    (1, 129, 256, 2, 16),     # one sequence one token past a 128-token column chunk
])
def test_backward_bf16_matches_oracle(B, T, d, K, D_h):
    _check_bf16_backward(*_bf16_backward_case(B, T, d, K, D_h, seed=B * 31 + T))


@pytest.mark.parametrize("B,T,d,K,D_h", [
    (3, 100, 256, 2, 32),     # narrow forward tiles
    (2, 2500, 512, 2, 32),    # wide forward tiles, tiles overlapping by the conv halo
    (50, 3, 256, 2, 32),      # sequences shorter than the conv
])
def test_backward_bf16_saved_kv_matches_oracle(B, T, d, K, D_h):
    """With ENGRAM_SAVE_KV the forward's k and v (fp32 accumulations of the
    bf16 products) replace the backward's recomputation: the same bounds
    hold."""
    _check_bf16_backward(*_bf16_backward_case(B, T, d, K, D_h, seed=B * 17 + T,
                                              flags=eg.SAVE_KV))


@pytest.mark.parametrize("B,T,d,flags", [
    (3, 100, 256, eg.NORM_SCALES),                 # narrow forward tiles
    (2, 2500, 512, eg.NORM_SCALES),                # wide forward tiles
    (2, 700, 256, eg.NORM_SCALES | eg.SAVE_KV),    # with k and v kept by the forward
])
def test_backward_bf16_norm_scales_match_oracle(B, T, d, flags):
    """Learnable RMSNorm scales on a bf16 layer: the gate weights h k by
    g_h g_k in the forward's pass K and in the backward's row kernel; the
    scales' gradients (after the conv weights' in dconv_w) are held with dh
    to the bf16 metric."""
    _check_bf16_backward(*_bf16_backward_case(B, T, d, 2, 32, seed=B * 7 + T, flags=flags))


@pytest.mark.parametrize("B,T,d,flags", [
    (3, 100, 256, eg.CONV_DILATED),                 # narrow forward tiles
    (2, 2500, 512, eg.CONV_DILATED),                # wide forward tiles, chunks inside sequences
    (40, 7, 256, eg.CONV_DILATED),                  # sequences shorter than the dilated taps
    (1, 300, 256, eg.CONV_DILATED | eg.SAVE_KV),    # one sequence over three column chunks
    (3, 129, 768, eg.CONV_DILATED | eg.NORM_SCALES),
    (64, 1, 256, eg.CONV_DILATED),                  # one-token sequences
])
def test_backward_bf16_dilated_matches_oracle(B, T, d, flags):
    """The dilated conv (taps 3, 6 and 9 tokens back) on a bf16 layer: the
    column walk keeps nine tokens of history per feature and completes a
    token's dvt 9 tokens later (or at its sequence's end); every gradient is
    held to the same bounds as the plain conv's."""
    _check_bf16_backward(*_bf16_backward_case(B, T, d, 2, 32, seed=B * 5 + T, flags=flags))


@pytest.mark.parametrize("B,T,d,flags", [
    (3, 100, 256, eg.CONV_PRENORM),                                 # narrow forward tiles
    (2, 2500, 512, eg.CONV_PRENORM | eg.NORM_SCALES),               # g_v's gradient too
    (40, 7, 256, eg.CONV_PRENORM | eg.CONV_DILATED),                # short sequences, dilated
    (1, 300, 256, eg.CONV_PRENORM | eg.SAVE_KV),                    # kept k and v
    (3, 129, 768, eg.CONV_PRENORM | eg.CONV_DILATED | eg.NORM_SCALES),
    (64, 1, 256, eg.CONV_PRENORM),                                  # one-token sequences
])
def test_backward_bf16_prenorm_matches_oracle(B, T, d, flags):
    """The pre-conv RMSNorm on a bf16 layer: the column walk carries dc (the
    conv input's gradient) and the partial sums of <g_v dc, vt>; a row
    kernel forms dvt through the norm's backward, dv and dalpha; every
    gradient, g_v's included, is held to the same bounds as the plain
    conv's."""
    _check_bf16_backward(*_bf16_backward_case(B, T, d, 2, 32, seed=B * 3 + T, flags=flags))


def _check_bf16_backward(g, ref, idx, rows, D_h):
    for name in ("dh", "dconv_w"):
        err = max_rel_err(g[name].cpu().numpy(), ref[name])
        assert err <= TOL_BF16, (name, err)
    adk, adv, ae = np.abs(ref["dk"][:, 0, :]), np.abs(ref["dv"]), np.abs(ref["e"])
    assert _within_gemm_bound(g["dWk"].cpu().numpy()[0], ref["dWk"][0], adk.T @ ae)
    assert _within_gemm_bound(g["dWv"].cpu().numpy(), ref["dWv"], adv.T @ ae)
    assert _within_gemm_bound(g["de"].cpu().numpy(), ref["de"],
                              adk @ np.abs(ref["Wk_bf"][0]) + adv @ np.abs(ref["Wv_bf"]))
    # and in norm, all three within the bf16 tolerance
    for name in ("dWk", "dWv", "de"):
        a, b = g[name].cpu().numpy().reshape(ref[name].shape), ref[name]
        assert np.linalg.norm(a - b) <= TOL_BF16 * np.linalg.norm(b), name
    # the sparse table gradient: keys bit-exact, rows within the bf16
    # tolerance of the oracle's, and bit-exact against the deterministic
    # reduction applied to the GPU's own de
    keys_ref, rows_ref = O.table_grad_segments_fast(idx, ref["de"].astype(np.float32), rows, D_h)
    U = int(g["n_unique"].item())
    assert U == keys_ref.size
    assert np.array_equal(g["keys"][:U].cpu().numpy(), keys_ref)
    a = g["rows"][:U].cpu().numpy()
    assert np.linalg.norm(a - rows_ref) <= TOL_BF16 * np.linalg.norm(rows_ref)
    keys_own, rows_own = O.table_grad_segments_fast(idx, g["de"].cpu().numpy(), rows, D_h)
    assert np.array_equal(g["rows"][:U].cpu().numpy().view(np.uint32), rows_own.view(np.uint32))


@pytest.mark.parametrize("B,T", [(2, 300), (2, 2500)])
def test_backward_bf16_is_deterministic(B, T):
    """Two runs give the same bits.  At 5,000 tokens the weight-gradient GEMM
    cuts each output tile's token range into parts summed in a fixed order."""
    a, _, _, _, _ = _bf16_backward_case(B, T, 256, 2, 32, seed=9)
    b, _, _, _, _ = _bf16_backward_case(B, T, 256, 2, 32, seed=9)
    for name in ("dh", "dWk", "dWv", "dconv_w", "de"):
        assert torch.equal(a[name], b[name]), name
    U = int(a["n_unique"].item())
    assert torch.equal(a["rows"][:U], b["rows"][:U])


def test_backward_bf16_layer27b_full_size():
    """The 27B-shaped layer at full size (8 x 4,096 tokens, d 2,560, 16 heads
    x 80 dims, 5.7B-parameter table): forward then backward on the device,
    every gradient against the oracle's fp64 backward on the same bf16
    values, the table gradient's keys bit-exact and its sums bit-exact on the
    GPU's own de."""
    from tests.engram_cases import bf16_bits
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
    L.forward(idx)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(27)
    dout = torch.randn((w.N, 1, w.d), generator=gen, device="cuda")
    g = L.backward(idx, dout)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    # a second call gives the same bits (the weight gradients' token parts
    # are summed in a fixed order)
    g2 = L.backward(idx, dout)
    for name in ("dh", "dWk", "dWv", "de"):
        assert torch.equal(g[name], g2[name]), name
    del g2
    f64 = O.bf16_bits_to_f64
    e = f64(bf16_bits(L.e))
    Wk, Wv = f64(bf16_bits(dense["Wk"])), f64(bf16_bits(dense["Wv"]))
    ref = O.layer_backward(e, f64(bf16_bits(dense["h"])).reshape(w.N, 1, w.d), Wk, Wv,
                           dense["conv_w"].cpu().numpy(), w.T, dout.cpu().numpy())
    for name in ("dh", "dconv_w"):
        err = max_rel_err(g[name].cpu().numpy(), ref[name])
        assert err <= TOL_BF16, (name, err)
    adk, adv, ae = np.abs(ref["dk"][:, 0, :]), np.abs(ref["dv"]), np.abs(e)
    assert _within_gemm_bound(g["dWk"].cpu().numpy()[0], ref["dWk"][0], adk.T @ ae)
    assert _within_gemm_bound(g["dWv"].cpu().numpy(), ref["dWv"], adv.T @ ae)
    assert _within_gemm_bound(g["de"].cpu().numpy(), ref["de"],
                              adk @ np.abs(Wk[0]) + adv @ np.abs(Wv))
    keys_ref, _ = O.table_grad_segments_fast(idx_ref, ref["de"].astype(np.float32), w.rows, w.D_h)
    U = int(g["n_unique"].item())
    assert U == keys_ref.size
    assert np.array_equal(g["keys"][:U].cpu().numpy(), keys_ref)
    _, rows_own = O.table_grad_segments_fast(idx_ref, g["de"].cpu().numpy(), w.rows, w.D_h)
    assert np.array_equal(g["rows"][:U].cpu().numpy().view(np.uint32), rows_own.view(np.uint32))
    del table, dense, L, g
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,T,d,E_heads", [(3, 100, 256, 2), (2, 2500, 512, 2)])
def test_forward_saved_kv(B, T, d, E_heads):
    """ENGRAM_SAVE_KV leaves out, alpha and e bit for bit as they are without
    it, and the saved k = W_k e and v = W_v e are the fp32 accumulations of
    the bf16 products (exact in fp32): within the worst-case error of an
    E-term fp32 sum, E 2^-24 times the sum of the absolute products, of the
    oracle's fp64 contractions."""
    from tests.engram_cases import bf16_bits, bf16_dev
    rng = np.random.default_rng(B * 7 + T)
    K, D_h = E_heads, 32
    J, E, N = 2 * K, 2 * K * D_h, B * T
    rows = synth.primes_at_most(2003, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    h = rng.standard_normal((B, T, 1, d)).astype(np.float32)
    conv_w = (rng.standard_normal((d, 4)) * 0.5).astype(np.float32)
    idx = dev(np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32).reshape(B, T, J))
    outs = []
    for flags in (0, eg.SAVE_KV):
        cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64),
                          flags=flags)
        L = Layer(cfg, B, T, packed_table(tables, "bf16"), bf16_dev(h), bf16_dev(Wk),
                  bf16_dev(Wv), dev(conv_w), torch.bfloat16)
        L.forward(idx)
        torch.cuda.synchronize()
        assert eg.engram_get_status() == 0
        outs.append(L)
    plain, kept = outs
    assert eg.engram_saved_size(kept.cfg, N) == ((N * 4 + 255) // 256) * 256 + N * 2 * d * 4
    assert torch.equal(plain.out, kept.out)
    assert torch.equal(plain.e, kept.e)
    assert torch.equal(plain.saved[: N * 4], kept.saved[: N * 4])
    off = ((N * 4 + 255) // 256) * 256
    kv = kept.saved[off: off + N * 2 * d * 4].view(torch.float32).reshape(N, 2 * d).cpu().numpy()
    f64 = O.bf16_bits_to_f64
    e64 = f64(bf16_bits(kept.e))
    wk64 = f64(synth.to_bf16_bits(Wk))[0]
    wv64 = f64(synth.to_bf16_bits(Wv))
    for got, W in ((kv[:, :d], wk64), (kv[:, d:], wv64)):
        want = e64 @ W.T
        bound = np.abs(e64) @ np.abs(W).T
        assert float(np.max(np.abs(got - want) - E * 2.0 ** -24 * bound)) <= 0.0


def test_backward_bf16_on_two_streams_at_once():
    """Two layers' bf16 backwards issued on two CUDA streams with no
    synchronisation between them give the same bits as each run alone.  The
    weight-gradient GEMM cuts each output tile's 8,192-token range into
    parts that wait for one another, so its CTAs must all be resident
    together; two such grids do not fit the GPU at once."""
    from tests.engram_cases import bf16_dev
    B, T, d, K, D_h = 2, 4096, 1024, 2, 128
    J, E, N = 2 * K, 2 * K * D_h, B * T
    rows = synth.primes_at_most(2003, J)
    layers, idxs, douts = [], [], []
    for seed in (31, 32):
        rng = np.random.default_rng(seed)
        cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((J, 3), np.uint64))
        tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
        L = Layer(cfg, B, T, packed_table(tables, "bf16"),
                  bf16_dev(rng.standard_normal((B, T, 1, d)).astype(np.float32)),
                  bf16_dev((rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)),
                  bf16_dev((rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)),
                  dev((rng.standard_normal((d, 4)) * 0.5).astype(np.float32)), torch.bfloat16)
        idx = dev(np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32)
                  .reshape(B, T, J))
        L.forward(idx)
        layers.append(L)
        idxs.append(idx)
        douts.append(dev(rng.standard_normal((N, 1, d)).astype(np.float32)))
    torch.cuda.synchronize()
    alone = [layers[i].backward(idxs[i], douts[i]) for i in range(2)]
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    streams = (torch.cuda.Stream(), torch.cuda.Stream())
    both = []
    for i in range(2):
        with torch.cuda.stream(streams[i]):  # buffers and calls on stream i
            both.append(layers[i].backward(idxs[i], douts[i]))
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    for i in range(2):
        for name in ("dh", "dWk", "dWv", "dconv_w", "de", "n_unique"):
            assert torch.equal(both[i][name], alone[i][name]), (i, name)
        U = int(alone[i]["n_unique"].item())
        assert torch.equal(both[i]["keys"][:U], alone[i]["keys"][:U])
        assert torch.equal(both[i]["rows"][:U], alone[i]["rows"][:U])
