"""Parity of the formulation variants (conv dilation 3, pre-conv RMSNorm,
per-branch conv, learnable RMSNorm scales) of the fp32 layer with the
oracle: forward, decode streaming and every gradient, including the
small-parameter block's, within the fp32 tolerance (1e-5 max relative
error with a 1e-3 RMS floor); bf16 layers with the scales, the dilated conv
and the pre-conv norm against the bf16 metric; bf16 layers refuse more than
one branch."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O
from tests.engram_cases import dev, max_rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-5
DIL, PRE, BR, SC = eg.CONV_DILATED, eg.CONV_PRENORM, eg.CONV_PER_BRANCH, eg.NORM_SCALES
FLAG_SETS = [DIL, PRE, BR, SC, PRE | SC, DIL | PRE | BR | SC]


def _ws(nbytes):
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device="cuda")


def _layer(seed, flags, B=2, T=13, M=2, d=64, K=2, D_h=8):
    rng = np.random.default_rng(seed)
    J, E, N = 2 * K, 2 * K * D_h, B * T
    rows = synth.primes_at_most(101, J)
    cfg = eg.make_cfg(K, D_h, d, M, 1000, 770, eg.F32, rows, np.ones((J, 3), np.uint64),
                      flags=flags)
    n_par = eg.engram_param_floats(cfg)
    assert n_par == O.param_count(flags, M, d)
    block = (rng.standard_normal(n_par) * 0.5).astype(np.float32)
    if flags & SC:
        n_conv = (M if flags & BR else 1) * d * 4
        block[n_conv:] = (1.0 + 0.3 * rng.standard_normal(n_par - n_conv)).astype(np.float32)
    x = dict(
        e=rng.standard_normal((N, E)).astype(np.float32),
        h=rng.standard_normal((N, M, d)).astype(np.float32),
        Wk=(rng.standard_normal((M, d, E)) / np.sqrt(E)).astype(np.float32),
        Wv=(rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32),
        block=block,
        dout=rng.standard_normal((N, M, d)).astype(np.float32),
        idx=np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32),
    )
    return cfg, x, B, T, M, d, E, J, D_h


@pytest.mark.parametrize("flags", FLAG_SETS)
def test_variant_forward_and_backward_match_oracle(flags):
    cfg, x, B, T, M, d, E, J, D_h = _layer(100 + flags, flags)
    N = B * T
    e, h = dev(x["e"]), dev(x["h"])
    Wk, Wv, block = dev(x["Wk"]), dev(x["Wv"]), dev(x["block"])
    out = torch.empty((N, M, d), device="cuda")
    saved = _ws(eg.engram_saved_size(cfg, N))
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    eg.engram_forward(cfg, None, None, e, h, Wk, Wv, block, None, out, saved, B, T, _ws(fb), fb)
    ref = O.layer_forward_v(x["e"], x["h"], x["Wk"], x["Wv"], x["block"], T, flags)
    assert max_rel_err(out.cpu().numpy(), ref["out"]) <= TOL
    g = dict(dh=torch.empty((N, M, d), device="cuda"), dWk=torch.empty((M, d, E), device="cuda"),
             dWv=torch.empty((d, E), device="cuda"),
             dblock=torch.full((block.numel(),), 7.0, device="cuda"),
             de=torch.empty((N, E), device="cuda"))
    keys = torch.empty(N * J, dtype=torch.int64, device="cuda")
    rows_out = torch.empty((N * J, D_h), device="cuda")
    nu = torch.zeros(1, dtype=torch.int32, device="cuda")
    bb = eg.engram_workspace_size(cfg, eg.WS_BACKWARD, N)
    eg.engram_backward(cfg, dev(x["idx"]), e, h, Wk, Wv, block, saved, dev(x["dout"]), g["dh"],
                       g["dWk"], g["dWv"], g["dblock"], g["de"], keys, rows_out, nu, B, T,
                       _ws(bb), bb)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    want = O.layer_backward_v(x["e"], x["h"], x["Wk"], x["Wv"], x["block"], T, x["dout"], flags)
    for name in ("dh", "dWk", "dWv", "de", "dblock"):
        err = max_rel_err(g[name].cpu().numpy(), want[name])
        assert err <= TOL, (name, err)


@pytest.mark.parametrize("flags", FLAG_SETS)
def test_variant_decode_streaming_matches_whole_sequences(flags):
    cfg, x, B, T, M, d, E, J, D_h = _layer(200 + flags, flags, T=12)
    dil = 3 if flags & DIL else 1
    ref = O.layer_forward_v(x["e"], x["h"], x["Wk"], x["Wv"], x["block"], T, flags)
    eb = x["e"].reshape(B, T, E)
    hb = x["h"].reshape(B, T, M, d)
    state = torch.zeros((B, M, 3 * dil, d), device="cuda")
    Wk, Wv, block = dev(x["Wk"]), dev(x["Wv"]), dev(x["block"])
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, B)
    ws = _ws(fb)
    out = torch.empty((B, 1, M, d), device="cuda")
    got = []
    for t in range(T):
        eg.engram_forward(cfg, None, None, dev(np.ascontiguousarray(eb[:, t])),
                          dev(np.ascontiguousarray(hb[:, t])), Wk, Wv, block, state, out, None,
                          B, 1, ws, fb)
        got.append(out[:, 0].cpu().numpy().copy())
    got = np.stack(got, axis=1).reshape(B * T, M, d)
    # The state carries the conv inputs between steps in fp32 (the API's state
    # type): each is rounded once (relative 2^-24), so out differs from the
    # whole-sequence forward by at most SiLU' (< 1.1) times the conv of those
    # roundings, plus out's own rounding; twice that is allowed.
    P = O.unpack_params(x["block"], flags, M, d)
    conv_abs = O.causal_conv_v(np.abs(ref["c"]), np.abs(P["w"]), T, dil)
    bound = 2.0 ** -23 * (np.abs(ref["out"]) + 1.1 * conv_abs)
    assert np.all(np.abs(got - ref["out"]) <= bound), float(np.max(np.abs(got - ref["out"]) - bound))
    assert eg.engram_get_status() == 0


def test_bf16_layers_refuse_two_branches():
    K, D_h, d = 2, 32, 256
    rows = synth.primes_at_most(1009, 2 * K)
    cfg = eg.make_cfg(K, D_h, d, 2, 1000, 770, eg.BF16, rows, np.ones((2 * K, 3), np.uint64),
                      flags=eg.CONV_PRENORM)
    N, E = 4, 2 * K * D_h
    e = torch.zeros((N, E), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((N, d), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((d, E), dtype=torch.bfloat16, device="cuda")
    cw = torch.zeros((d, 4), device="cuda")
    out = torch.empty_like(h)
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    with pytest.raises(eg.EngramError) as ex:
        eg.engram_forward(cfg, None, None, e, h, W, W, cw, None, out, None, 1, N, _ws(fb), fb)
    assert eg.ERRORS[ex.value.rc] == "ENGRAM_ERR_UNSUPPORTED"


@pytest.mark.parametrize("N,T", [(300, 100), (5000, 2500)])
def test_bf16_norm_scales_forward_matches_oracle(N, T):
    """bf16 layer with learnable RMSNorm scales: out within the bf16 metric
    of the oracle's fp64 forward on the same bf16 values, alpha to 1e-5."""
    from tests.engram_cases import bf16_dev
    rng = np.random.default_rng(N)
    K, D_h, d = 2, 32, 256
    E = 2 * K * D_h
    rows = synth.primes_at_most(1009, 2 * K)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((2 * K, 3), np.uint64),
                      flags=eg.NORM_SCALES)
    e = rng.standard_normal((N, E)).astype(np.float32)
    h = rng.standard_normal((N, 1, d)).astype(np.float32)
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    block = np.r_[(rng.standard_normal(4 * d) * 0.5), 1.0 + 0.3 * rng.standard_normal(2 * d)]
    block = block.astype(np.float32)
    assert eg.engram_param_floats(cfg) == block.size
    out = torch.empty((N, 1, d), dtype=torch.bfloat16, device="cuda")
    saved = _ws(eg.engram_saved_size(cfg, N))
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    eg.engram_forward(cfg, None, None, bf16_dev(e), bf16_dev(h), bf16_dev(Wk), bf16_dev(Wv),
                      dev(block), None, out, saved, N // T, T, _ws(fb), fb)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    f64 = O.bf16_bits_to_f64
    b = synth.to_bf16_bits
    ref = O.layer_forward_v(f64(b(e)), f64(b(h)), f64(b(Wk)), f64(b(Wv)), block, T, eg.NORM_SCALES)
    assert max_rel_err(out.float().cpu().numpy(), ref["out"]) <= 2e-2
    alpha = saved[: N * 4].view(torch.float32).cpu().numpy()
    assert np.max(np.abs(alpha - ref["alpha"].reshape(-1))) <= 1e-5


@pytest.mark.parametrize("B,T,d", [(3, 100, 256), (2, 2500, 512), (40, 7, 256), (1, 4100, 256)])
def test_bf16_dilated_forward_matches_oracle(B, T, d):
    """bf16 layer with the dilated conv (taps at t, t-3, t-6, t-9): out within
    the bf16 metric of the oracle; narrow and wide tiles, sequences shorter
    than the conv's 9-token history, tile seams (tiles overlap by 9)."""
    from tests.engram_cases import bf16_dev
    rng = np.random.default_rng(B * 13 + T)
    K, D_h = 2, 32
    E, N = 2 * K * D_h, B * T
    rows = synth.primes_at_most(1009, 2 * K)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((2 * K, 3), np.uint64),
                      flags=eg.CONV_DILATED)
    e = rng.standard_normal((N, E)).astype(np.float32)
    h = rng.standard_normal((N, 1, d)).astype(np.float32)
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    block = (rng.standard_normal(4 * d) * 0.5).astype(np.float32)
    out = torch.empty((N, 1, d), dtype=torch.bfloat16, device="cuda")
    saved = _ws(eg.engram_saved_size(cfg, N))
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    eg.engram_forward(cfg, None, None, bf16_dev(e), bf16_dev(h), bf16_dev(Wk), bf16_dev(Wv),
                      dev(block), None, out, saved, B, T, _ws(fb), fb)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    f64 = O.bf16_bits_to_f64
    b = synth.to_bf16_bits
    ref = O.layer_forward_v(f64(b(e)), f64(b(h)), f64(b(Wk)), f64(b(Wv)), block, T,
                            eg.CONV_DILATED)
    assert max_rel_err(out.float().cpu().numpy(), ref["out"]) <= 2e-2


def _bf16_block(rng, cfg, d):
    """conv weights N(0, 0.5^2), then the norm scales 1 + N(0, 0.3^2)."""
    n = eg.engram_param_floats(cfg)
    block = rng.standard_normal(n) * 0.5
    block[4 * d:] = 1.0 + 0.3 * rng.standard_normal(n - 4 * d)
    return block.astype(np.float32)


@pytest.mark.parametrize("B,T,d,flags", [
    (3, 100, 256, PRE),              # narrow forward tiles
    (2, 2500, 512, PRE | SC),        # wide tiles, g_v with the other scales
    (40, 7, 256, PRE | DIL),         # sequences shorter than the dilated taps
    (1, 4100, 256, PRE | DIL | SC),  # one sequence over many conv chunks
    (2, 700, 256, PRE | eg.SAVE_KV), # v written into the kept [k | v] rows
])
def test_bf16_prenorm_forward_matches_oracle(B, T, d, flags):
    """bf16 layer with the pre-conv RMSNorm (c = RMSNorm(alpha v) g_v): out
    within the bf16 metric of the oracle's fp64 forward on the same bf16
    values, alpha to 1e-5, and with ENGRAM_SAVE_KV the kept k and v against
    the oracle's."""
    from tests.engram_cases import bf16_dev
    rng = np.random.default_rng(B * 11 + T + flags)
    K, D_h = 2, 32
    E, N = 2 * K * D_h, B * T
    rows = synth.primes_at_most(1009, 2 * K)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((2 * K, 3), np.uint64),
                      flags=flags)
    e = rng.standard_normal((N, E)).astype(np.float32)
    h = rng.standard_normal((N, 1, d)).astype(np.float32)
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    block = _bf16_block(rng, cfg, d)
    vflags = flags & (PRE | DIL | SC)
    assert block.size == O.param_count(vflags, 1, d)
    out = torch.empty((N, 1, d), dtype=torch.bfloat16, device="cuda")
    saved = _ws(eg.engram_saved_size(cfg, N))
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    eg.engram_forward(cfg, None, None, bf16_dev(e), bf16_dev(h), bf16_dev(Wk), bf16_dev(Wv),
                      dev(block), None, out, saved, B, T, _ws(fb), fb)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    f64 = O.bf16_bits_to_f64
    b = synth.to_bf16_bits
    ref = O.layer_forward_v(f64(b(e)), f64(b(h)), f64(b(Wk)), f64(b(Wv)), block, T, vflags)
    assert max_rel_err(out.float().cpu().numpy(), ref["out"]) <= 2e-2
    alpha = saved[: N * 4].view(torch.float32).cpu().numpy()
    assert np.max(np.abs(alpha - ref["alpha"].reshape(-1))) <= 1e-5
    if flags & eg.SAVE_KV:
        off = (N * 4 + 255) // 256 * 256
        kv = saved[off: off + N * 2 * d * 4].view(torch.float32).reshape(N, 2 * d).cpu().numpy()
        assert max_rel_err(kv[:, :d], ref["k"][:, 0]) <= 1e-3
        assert max_rel_err(kv[:, d:], ref["v"]) <= 1e-3


@pytest.mark.parametrize("flags,D_h", [
    (DIL, 32), (PRE, 32), (PRE | DIL | SC, 32),
    (DIL, 128), (SC, 128), (DIL | SC, 128),   # E = 512: split units (K in two halves per tile)
])
def test_bf16_decode_matches_whole_sequences(flags, D_h):
    """Decode steps of a bf16 layer (conv state [B, 1, 3 dil, d], the conv
    inputs of the previous steps: vt, or RMSNorm(vt) g_v with the pre-conv
    norm) against the oracle's whole-sequence forward, each step within the
    bf16 metric."""
    from tests.engram_cases import bf16_dev
    rng = np.random.default_rng(70 + flags + D_h)
    B, T, K, d = 24, 14, 2, 256
    E = 2 * K * D_h
    rows = synth.primes_at_most(1009, 2 * K)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((2 * K, 3), np.uint64),
                      flags=flags)
    e = rng.standard_normal((B, T, E)).astype(np.float32)
    h = rng.standard_normal((B, T, 1, d)).astype(np.float32)
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    block = _bf16_block(rng, cfg, d)
    f64 = O.bf16_bits_to_f64
    b = synth.to_bf16_bits
    ref = O.layer_forward_v(f64(b(e)).reshape(B * T, E), f64(b(h)).reshape(B * T, 1, d),
                            f64(b(Wk)), f64(b(Wv)), block, T, flags)
    ref_out = ref["out"].reshape(B, T, 1, d)
    state = torch.zeros((B, 1, 3 * O.dilation_of(flags), d), device="cuda")
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, B)
    ws = _ws(fb)
    Wk_d, Wv_d, blk = bf16_dev(Wk), bf16_dev(Wv), dev(block)
    out = torch.empty((B, 1, 1, d), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        eg.engram_forward(cfg, None, None, bf16_dev(np.ascontiguousarray(e[:, t])),
                          bf16_dev(np.ascontiguousarray(h[:, t])), Wk_d, Wv_d, blk, state, out,
                          None, B, 1, ws, fb)
        got = out[:, 0].float().cpu().numpy()
        assert max_rel_err(got, ref_out[:, t]) <= 2e-2, t
    assert eg.engram_get_status() == 0
