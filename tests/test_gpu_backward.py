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
