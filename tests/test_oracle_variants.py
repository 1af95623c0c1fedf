"""Pins of the oracle's formulation variants (conv dilation, pre-conv RMSNorm,
per-branch conv, learnable RMSNorm scales): with no flag they are the base
layer; special cases reduce to simpler ones; decode streaming equals the
whole-sequence forward; every gradient matches central finite differences.
CPU only."""
import itertools

import numpy as np
import pytest

from oracle import engram_oracle as O

DIL, PRE, BR, SC = O.CONV_DILATED, O.CONV_PRENORM, O.CONV_PER_BRANCH, O.NORM_SCALES
FLAG_SETS = [DIL, PRE, BR, SC, PRE | SC, DIL | PRE | BR | SC]


def _case(seed, B=2, T=12, M=2, d=8, E=12, flags=0):
    rng = np.random.default_rng(seed)
    N = B * T
    e = rng.standard_normal((N, E))
    h = rng.standard_normal((N, M, d))
    Wk = rng.standard_normal((M, d, E)) / np.sqrt(E)
    Wv = rng.standard_normal((d, E)) / np.sqrt(E)
    block = rng.standard_normal(O.param_count(flags, M, d)) * 0.5
    if flags & SC:  # scales near one
        n_conv = (M if flags & BR else 1) * d * 4
        block[n_conv:] = 1.0 + 0.3 * rng.standard_normal(block.size - n_conv)
    dout = rng.standard_normal((N, M, d))
    return e, h, Wk, Wv, block, T, dout


def test_no_flag_is_the_base_layer():
    e, h, Wk, Wv, block, T, dout = _case(1)
    a = O.layer_forward(e, h, Wk, Wv, block.reshape(-1, 4), T)
    b = O.layer_forward_v(e, h, Wk, Wv, block, T, 0)
    for name in ("out", "alpha", "y", "vt"):
        assert np.array_equal(a[name], b[name]), name
    ga = O.layer_backward(e, h, Wk, Wv, block.reshape(-1, 4), T, dout)
    gb = O.layer_backward_v(e, h, Wk, Wv, block, T, dout, 0)
    for name in ("dh", "dWk", "dWv", "de"):
        assert np.allclose(ga[name], gb[name], rtol=1e-12, atol=1e-12), name
    assert np.allclose(ga["dconv_w"].reshape(-1), gb["dblock"], rtol=1e-12, atol=1e-12)


def test_unit_scales_and_equal_branch_convs_change_nothing():
    M, d = 3, 8
    e, h, Wk, Wv, block, T, dout = _case(2, M=M, d=d)
    base = O.layer_forward_v(e, h, Wk, Wv, block, T, PRE)
    ones = np.concatenate([block, np.ones(3 * M * d)])
    scaled = O.layer_forward_v(e, h, Wk, Wv, ones, T, PRE | SC)
    assert np.array_equal(base["out"], scaled["out"])
    per_branch = np.tile(block, M)  # every branch gets the shared weights
    br = O.layer_forward_v(e, h, Wk, Wv, per_branch, T, PRE | BR)
    assert np.array_equal(base["out"], br["out"])


def test_dilated_conv_taps_and_short_sequences():
    e, h, Wk, Wv, block, T, dout = _case(3, B=3, T=3, M=1)
    f = O.layer_forward_v(e, h, Wk, Wv, block, 3, DIL)
    # every earlier tap lies 3, 6 or 9 tokens back: outside sequences of 3
    w = block.reshape(1, -1, 4)
    assert np.allclose(f["y"], w[None, :, :, 3] * f["vt"], rtol=0, atol=1e-15)
    # an impulse in c shows up 0, 3, 6, 9 tokens later, with the reversed taps
    c = np.zeros((20, 1, 8))
    c[2, 0, :] = 1.0
    y = O.causal_conv_v(c, w, 20, 3)
    for lag, i in zip((0, 3, 6, 9), (3, 2, 1, 0)):
        assert np.array_equal(y[2 + lag, 0], w[0, :, i])
    others = [t for t in range(20) if t not in (2, 5, 8, 11)]
    assert not y[others].any()


@pytest.mark.parametrize("T", [1, 2, 3, 7, 12, 20])
def test_dilated_conv_is_three_interleaved_plain_convs(T):
    """Taps 3, 6 and 9 tokens back only ever read tokens of the same residue
    mod 3 within a sequence, so the dilated conv equals three independent
    dilation-1 convs, one over each residue's subsequence (bit for bit: the
    same terms in the same order)."""
    rng = np.random.default_rng(T)
    B, d = 3, 5
    c = rng.standard_normal((B * T, 1, d))
    w = rng.standard_normal((1, d, 4))
    y = O.causal_conv_v(c, w, T, 3)
    for b in range(B):
        for r in range(3):
            rows = np.arange(b * T + r, (b + 1) * T, 3)
            if rows.size == 0:
                continue
            sub = O.causal_conv_v(c[rows], w, rows.size, 1)
            assert np.array_equal(y[rows], sub), (b, r)


@pytest.mark.parametrize("flags", FLAG_SETS)
def test_decode_streaming_equals_whole_sequences(flags):
    B, T, M, d = 2, 12, 2, 8
    e, h, Wk, Wv, block, _, _ = _case(4 + flags, B=B, T=T, M=M, d=d, flags=flags)
    whole = O.layer_forward_v(e, h, Wk, Wv, block, T, flags)
    dil = O.dilation_of(flags)
    st = np.zeros((B, M, 3 * dil, d))
    eb, hb = e.reshape(B, T, -1), h.reshape(B, T, M, d)
    out_w = whole["out"].reshape(B, T, M, d)
    for t in range(T):
        out, alpha, st = O.decode_step_v(eb[:, t], hb[:, t], Wk, Wv, block, st, flags)
        assert np.allclose(out, out_w[:, t], rtol=1e-12, atol=1e-12), t
        assert np.allclose(alpha, whole["alpha"].reshape(B, T, M)[:, t], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("flags", FLAG_SETS)
def test_variant_gradients_match_finite_differences(flags):
    e, h, Wk, Wv, block, T, dout = _case(10 + flags, flags=flags)
    g = O.layer_backward_v(e, h, Wk, Wv, block, T, dout, flags)

    def loss(e_, h_, Wk_, Wv_, b_):
        return float(np.sum(dout * O.layer_forward_v(e_, h_, Wk_, Wv_, b_, T, flags)["out"]))

    rng = np.random.default_rng(flags)
    args = [e, h, Wk, Wv, block]
    names = ["de", "dh", "dWk", "dWv", "dblock"]
    eps = 1e-6
    for a, name in enumerate(names):
        x = args[a]
        flat = x.reshape(-1)
        picks = rng.choice(flat.size, size=min(12, flat.size), replace=False)
        if name == "dblock":  # every scale group and every conv tap at least once
            picks = np.unique(np.r_[picks, np.arange(0, flat.size, max(1, flat.size // 16))])
        for p in picks:
            old = flat[p]
            flat[p] = old + eps
            lp = loss(*args)
            flat[p] = old - eps
            lm = loss(*args)
            flat[p] = old
            fd = (lp - lm) / (2 * eps)
            got = g[name].reshape(-1)[p]
            assert abs(got - fd) <= 1e-6 * max(1.0, abs(fd)), (name, p, got, fd)


def test_a_planted_mistake_fails_the_pins():
    """Dropping the pre-conv norm's backward (treating c as vt) must be seen."""
    flags = PRE
    e, h, Wk, Wv, block, T, dout = _case(31, flags=flags)
    g = O.layer_backward_v(e, h, Wk, Wv, block, T, dout, flags)
    wrong = O.layer_backward_v(e, h, Wk, Wv, block, T, dout, 0)
    assert not np.allclose(g["dh"], wrong["dh"], rtol=1e-3)


def test_param_counts():
    for M, d in itertools.product((1, 3), (8, 64)):
        assert O.param_count(0, M, d) == 4 * d
        assert O.param_count(BR, M, d) == 4 * d * M
        assert O.param_count(SC, M, d) == 4 * d + 2 * M * d
        assert O.param_count(SC | PRE | BR, M, d) == 4 * d * M + 3 * M * d
