"""Pins of the oracle's backward pass: central finite differences in fp64 for
every parameter group, and the sparse table gradient's reduction order.
CPU only."""
import numpy as np
import pytest

from oracle import engram_oracle as O
from hashed_gram_conditional_engram_b200 import synth

STEP = 1e-5
TOL = 1e-6


def _loss(e, h, Wk, Wv, w, T, u):
    return float(np.sum(u * O.layer_forward(e, h, Wk, Wv, w, T)["out"]))


def _check(name, arr, grad, f, rng, n=24):
    """Central differences at n random entries of `arr` (perturbed in place)."""
    scale = max(float(np.sqrt(np.mean(grad ** 2))), 1e-12)
    flat = arr.reshape(-1)
    gflat = grad.reshape(-1)
    for i in rng.choice(flat.size, size=min(n, flat.size), replace=False):
        old = flat[i]
        flat[i] = old + STEP
        fp = f()
        flat[i] = old - STEP
        fm = f()
        flat[i] = old
        fd = (fp - fm) / (2 * STEP)
        assert abs(fd - gflat[i]) <= TOL * max(abs(gflat[i]), scale), (name, i, fd, gflat[i])


@pytest.mark.parametrize("M", [1, 4])
def test_finite_differences_all_groups(M):
    w_ = synth.workload("tiny")
    rng = np.random.default_rng(10 + M)
    inp = synth.host_inputs(w_)
    proj, V_c = O.build_vocab_proj(inp["keys"])
    idx = O.hash_indices(proj, inp["ids"], inp["mult"], inp["rows"], w_.K, V_c).reshape(-1, w_.J)
    tables = [t.astype(np.float64) for t in inp["tables"]]
    T = w_.T
    N = w_.N
    h = rng.standard_normal((N, M, w_.d))
    Wk = rng.standard_normal((M, w_.d, w_.E)) * 0.3
    Wv = rng.standard_normal((w_.d, w_.E)) * 0.3
    w = rng.standard_normal((w_.d, 4)) * 0.5
    u = rng.standard_normal((N, M, w_.d))

    def e_of():
        return O.gather(idx, tables)

    e = e_of()
    g = O.layer_backward(e, h, Wk, Wv, w, T, u)
    f = lambda: _loss(e_of(), h, Wk, Wv, w, T, u)
    _check("h", h, g["dh"], f, rng)
    _check("Wk", Wk, g["dWk"], f, rng)
    _check("Wv", Wv, g["dWv"], f, rng)
    _check("conv_w", w, g["dconv_w"], f, rng)
    # table rows through the gather: the dense scatter of de is the gradient
    dT = O.table_grad_f64(idx, g["de"], w_.rows, w_.D_h)
    for j in range(w_.J):
        touched = np.unique(idx[:, j])
        sel = rng.choice(touched, size=min(3, touched.size), replace=False)
        for s in sel:
            for c in rng.choice(w_.D_h, size=3, replace=False):
                old = tables[j][s, c]
                tables[j][s, c] = old + STEP
                fp = f()
                tables[j][s, c] = old - STEP
                fm = f()
                tables[j][s, c] = old
                fd = (fp - fm) / (2 * STEP)
                scale = float(np.sqrt(np.mean(dT[j][touched] ** 2)))
                assert abs(fd - dT[j][s, c]) <= TOL * max(abs(dT[j][s, c]), scale)
        # an untouched row has zero gradient
        untouched = np.setdiff1d(np.arange(w_.rows[j]), touched)
        assert not dT[j][untouched].any()


def test_finite_differences_two_layer_chain():
    """The training workload: Engram at two layers (4 branches each), the
    second fed by the first; dh of layer 6 is the output gradient of layer 2."""
    w_ = synth.workload("train")
    rng = np.random.default_rng(21)
    L = [synth.host_inputs(w_, layer=l) for l in (2, 6)]
    E = []
    for inp in L:
        proj, V_c = O.build_vocab_proj(inp["keys"])
        idx = O.hash_indices(proj, inp["ids"], inp["mult"], inp["rows"], w_.K, V_c).reshape(-1, w_.J)
        E.append(O.gather(idx, [t.astype(np.float64) for t in inp["tables"]]))
    h0 = L[0]["h"].reshape(-1, w_.M, w_.d).astype(np.float64)
    u = L[0]["dout"].reshape(-1, w_.M, w_.d).astype(np.float64)
    P = [[inp["Wk"].astype(np.float64), inp["Wv"].astype(np.float64),
          inp["conv_w"].astype(np.float64)] for inp in L]

    def loss():
        h1 = O.layer_forward(E[0], h0, *P[0], w_.T)["out"]
        h2 = O.layer_forward(E[1], h1, *P[1], w_.T)["out"]
        return float(np.sum(u * h2))

    h1 = O.layer_forward(E[0], h0, *P[0], w_.T)["out"]
    g6 = O.layer_backward(E[1], h1, *P[1], w_.T, u)
    g2 = O.layer_backward(E[0], h0, *P[0], w_.T, g6["dh"])
    _check("h0", h0, g2["dh"], loss, rng)
    _check("Wk2", P[0][0], g2["dWk"], loss, rng)
    _check("Wv2", P[0][1], g2["dWv"], loss, rng)
    _check("w2", P[0][2], g2["dconv_w"], loss, rng)
    _check("Wk6", P[1][0], g6["dWk"], loss, rng)
    _check("Wv6", P[1][1], g6["dWv"], loss, rng)
    _check("w6", P[1][2], g6["dconv_w"], loss, rng)


def test_segment_sum_order_is_ascending_token():
    # three tokens hit the same row with de values 1e8, -1e8, 1 (fp32):
    # ascending order gives (1e8 - 1e8) + 1 = 1; any order that adds 1 to 1e8
    # first loses it (fp32 spacing at 1e8 is 8) and gives 0.
    rows = [5, 5]
    D_h = 1
    idx = np.array([[2, 0], [2, 1], [2, 3]], dtype=np.int32)
    de = np.array([[1e8, 0.0], [-1e8, 0.0], [1.0, 0.0]], dtype=np.float32)
    keys, grads = O.table_grad_segments(idx, de, rows, D_h)
    assert keys.tolist() == [2, 5, 6, 8]          # head 1's rows start at P_0 = 5
    assert grads[0, 0] == np.float32(1.0)
    k2, g2 = O.table_grad_segments_fast(idx, de, rows, D_h)
    assert np.array_equal(k2, keys) and np.array_equal(g2.view(np.uint32), grads.view(np.uint32))


def test_segment_sums_match_dense_scatter_and_fast_form():
    rng = np.random.default_rng(6)
    rows = [1009, 1013, 1019, 1021]
    D_h, N = 16, 500
    # Zipf-like skew: many tokens on few slots
    idx = np.stack([np.minimum(rng.zipf(1.3, N) - 1, p - 1) for p in rows], -1).astype(np.int32)
    de = rng.standard_normal((N, len(rows) * D_h)).astype(np.float32)
    keys, grads = O.table_grad_segments(idx, de, rows, D_h)
    k2, g2 = O.table_grad_segments_fast(idx, de, rows, D_h)
    assert np.array_equal(keys, k2)
    assert np.array_equal(grads.view(np.uint32), g2.view(np.uint32))
    assert np.all(np.diff(keys) > 0)
    base = np.concatenate([[0], np.cumsum(rows)[:-1]])
    assert keys.size == len({(j, int(s)) for j in range(len(rows)) for s in idx[:, j]})
    dense = O.table_grad_f64(idx, de.astype(np.float64), rows, D_h)
    for u, key in enumerate(keys.tolist()):
        j = int(np.searchsorted(base, key, side="right") - 1)
        s = key - base[j]
        cnt = int(np.sum(idx[:, j] == s))
        ref = dense[j][s]
        bound = cnt * 2 ** -23 * np.sum(np.abs(de[idx[:, j] == s][:, j * D_h:(j + 1) * D_h]), axis=0)
        assert np.all(np.abs(grads[u] - ref) <= bound + 1e-30)
