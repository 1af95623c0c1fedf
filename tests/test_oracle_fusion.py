"""Pins of the oracle's fusion steps (gate, value, conv, residual) against
closed forms, special cases and invariants.  CPU only."""
import math

import numpy as np
import torch

from oracle import engram_oracle as O
from hashed_gram_conditional_engram_b200 import synth


def _tiny(M=1, seed=0, T=64, B=1, d=64, E=64):
    rng = np.random.default_rng(seed)
    N = B * T
    e = rng.standard_normal((N, E)) * 0.02
    h = rng.standard_normal((N, M, d))
    Wk = rng.standard_normal((M, d, E)) * 0.5
    Wv = rng.standard_normal((d, E)) * 0.5
    w = rng.standard_normal((d, 4)) * 0.5
    return e, h, Wk, Wv, w, T


def test_zero_value_projection_returns_h_exactly():
    e, h, Wk, Wv, w, T = _tiny(M=2)
    r = O.layer_forward(e, h, Wk, np.zeros_like(Wv), w, T)
    assert np.array_equal(r["out"], h)
    # bf16 storage: out rounds h + 0 + SiLU(0) = h, which is already bf16
    hb = synth.to_bf16_bits(h.astype(np.float32))
    rb = O.layer_forward_bf16(synth.to_bf16_bits(e.astype(np.float32)), hb,
                              synth.to_bf16_bits(Wk.astype(np.float32)),
                              np.zeros(Wv.shape, np.uint16), w, T)
    assert np.array_equal(rb["out_bits"], hb)


def test_zero_key_projection_gives_half_gate():
    # k = 0 -> RMSNorm(k) = 0 -> z = 0 -> alpha = sigmoid(0) = 1/2 exactly
    e, h, Wk, Wv, w, T = _tiny(M=3)
    r = O.layer_forward(e, h, np.zeros_like(Wk), Wv, w, T)
    assert np.all(r["alpha"] == 0.5)


def test_gate_symmetry_under_key_negation():
    # alpha(-k) = sigmoid(-z) = 1 - alpha(k)
    e, h, Wk, Wv, w, T = _tiny(M=2)
    a = O.layer_forward(e, h, Wk, Wv, w, T)["alpha"]
    b = O.layer_forward(e, h, -Wk, Wv, w, T)["alpha"]
    assert np.allclose(a + b, 1.0, rtol=0, atol=1e-15)


def test_gate_closed_form_when_key_equals_hidden():
    # E = d, W_k = I and e = h give k = h: <h^, h^> = d * m / (m + eps) with
    # m = mean(h^2), so z = sqrt(d) * m / (m + eps)
    rng = np.random.default_rng(2)
    N, d = 10, 64
    h = rng.standard_normal((N, 1, d)) * rng.uniform(0.01, 3.0, size=(N, 1, 1))
    e = h[:, 0, :].copy()
    r = O.layer_forward(e, h, np.eye(d)[None], np.zeros((d, d)), np.zeros((d, 4)), N)
    m = np.mean(h[:, 0, :] ** 2, axis=-1)
    z = math.sqrt(d) * m / (m + O.RMS_EPS)
    assert np.allclose(r["alpha"][:, 0], 1.0 / (1.0 + np.exp(-z)), rtol=1e-14, atol=0)


def test_gate_orthogonal_key_gives_half():
    d = 8
    h = np.zeros((1, 1, d)); h[0, 0, 0] = 2.0
    e = np.zeros((1, d)); e[0, 1] = 3.0
    r = O.layer_forward(e, h, np.eye(d)[None], np.zeros((d, d)), np.zeros((d, 4)), 1)
    assert r["alpha"][0, 0] == 0.5


def test_gate_shrinks_with_disagreement():
    # larger disagreement between memory and context -> smaller alpha
    # (deepseek.club 二.1 (2): the gate factor falls as the two differ more)
    rng = np.random.default_rng(8)
    d = 32
    h = rng.standard_normal(d)
    noise = rng.standard_normal(d)
    alphas = []
    for mix in np.linspace(0.0, 1.0, 11):
        k = (1 - mix) * h + mix * (-h + 0.1 * noise)
        r = O.layer_forward(k[None], h[None, None], np.eye(d)[None], np.zeros((d, d)),
                            np.zeros((d, 4)), 1)
        alphas.append(r["alpha"][0, 0])
    assert all(a > b for a, b in zip(alphas, alphas[1:]))


def test_conv_impulse_response_and_sequence_boundary():
    # an impulse at t0 comes out as the reversed taps w[:,3], w[:,2], w[:,1], w[:,0]
    # at t0 .. t0+3, and never crosses into the next sequence
    T, d, M = 8, 5, 2
    rng = np.random.default_rng(1)
    w = rng.standard_normal((d, 4))
    for t0 in [0, 2, 5, 7]:
        vt = np.zeros((2 * T, M, d))
        vt[t0, 1, :] = 1.0
        y = O.causal_conv(vt, w, T)
        for t in range(2 * T):
            lag = t - t0
            want = w[:, 3 - lag] if 0 <= lag <= 3 and t < T else np.zeros(d)
            assert np.array_equal(y[t, 1], want), (t0, t)
            assert not y[t, 0].any()


def test_causality_hidden_state():
    e, h, Wk, Wv, w, T = _tiny(M=2)
    base = O.layer_forward(e, h, Wk, Wv, w, T)["out"]
    for t in [0, 17, 63]:
        h2 = h.copy()
        h2[t] += 1.0
        pert = O.layer_forward(e, h2, Wk, Wv, w, T)["out"]
        assert np.array_equal(base[:t], pert[:t])
        assert not np.array_equal(base[t], pert[t])


def test_causality_token_ids_through_full_pipeline():
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    proj, V_c = O.build_vocab_proj(inp["keys"])

    def run(ids):
        idx = O.hash_indices(proj, ids, inp["mult"], inp["rows"], w.K, V_c)
        e = O.gather(idx.reshape(-1, w.J), inp["tables"])
        return O.layer_forward(e, inp["h"].reshape(-1, w.M, w.d), inp["Wk"], inp["Wv"],
                               inp["conv_w"], w.T)["out"]

    base = run(inp["ids"])
    for t in [1, 30, 63]:
        ids = inp["ids"].copy()
        ids[0, t] = (ids[0, t] + 1) % w.V
        while proj[ids[0, t]] == proj[inp["ids"][0, t]]:
            ids[0, t] = (ids[0, t] + 1) % w.V
        pert = run(ids)
        assert np.array_equal(base[:t], pert[:t])
        assert not np.array_equal(base[t:], pert[t:])


def test_rmsnorm_of_constant_vector():
    x = np.full((1, 16), 3.0)
    assert np.allclose(O.rmsnorm(x), 3.0 / math.sqrt(9.0 + O.RMS_EPS), rtol=1e-15)


def test_sigmoid_silu_against_library():
    z = np.linspace(-30, 30, 601)
    zt = torch.tensor(z, dtype=torch.float64)
    assert np.allclose(O.sigmoid(z), torch.sigmoid(zt).numpy(), rtol=1e-14, atol=1e-300)
    assert np.allclose(O.silu(z), torch.nn.functional.silu(zt).numpy(), rtol=1e-13, atol=1e-300)


def test_bf16_rounding_against_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        (rng.standard_normal(1000) * 1e-39).astype(np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0,
                                  3.0e38], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f64_to_bf16_bits(x.astype(np.float64))
    assert np.array_equal(got, want)
    assert np.array_equal(O.bf16_bits_to_f64(want),
                          torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_decode_matches_sequence_forward():
    # stepping one token at a time with the rolling conv state reproduces the
    # whole-sequence forward
    e, h, Wk, Wv, w, _ = _tiny(M=2, T=9, B=3)
    B, T = 3, 9
    full = O.layer_forward(e, h, Wk, Wv, w, T)["out"].reshape(B, T, 2, -1)
    eb = e.reshape(B, T, -1)
    hb = h.reshape(B, T, 2, -1)
    st = np.zeros((B, 2, 3, h.shape[-1]))
    for t in range(T):
        out, _, st = O.decode_step(eb[:, t], hb[:, t], Wk, Wv, w, st)
        assert np.allclose(out, full[:, t], rtol=1e-13, atol=1e-13)


def test_multibranch_shares_value_and_conv():
    # branch m of a 2-branch layer equals a 1-branch layer with W_k = W_k[m]
    e, h, Wk, Wv, w, T = _tiny(M=2)
    both = O.layer_forward(e, h, Wk, Wv, w, T)["out"]
    for m in range(2):
        one = O.layer_forward(e, h[:, m:m + 1], Wk[m:m + 1], Wv, w, T)["out"]
        assert np.array_equal(both[:, m:m + 1], one)
