"""A seeded sweep of random shapes and formulation flags through the bf16
layer: forward and backward against the fp64 oracle (the same bounds as the
hand-picked cases), and decode streaming against the oracle's whole-sequence
forward.  The shapes mix one-token and short sequences, ragged tiles, narrow
and wide forward tiles (up to 10,000 tokens), every head count 2 K = 2 .. 16
and head widths 16 .. 128."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O
from tests.engram_cases import bf16_dev, dev, max_rel_err, ws
from tests.test_gpu_backward import _bf16_backward_case, _check_bf16_backward

pytestmark = pytest.mark.gpu

FLAG_SETS = [0, eg.SAVE_KV, eg.CONV_DILATED, eg.NORM_SCALES, eg.CONV_PRENORM,
             eg.CONV_DILATED | eg.NORM_SCALES | eg.SAVE_KV, eg.CONV_PRENORM | eg.CONV_DILATED]


def _layer_shapes(seed, n):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        d = int(rng.choice([256, 512, 768, 1024]))
        K = int(rng.integers(1, 9))
        D_h = int(rng.choice([16, 32, 48, 64, 80, 128]))
        if (2 * K * D_h) % 64:  # E a multiple of 64 (the tensor-core path's K step)
            continue
        B = int(rng.integers(1, 6))
        T = int(rng.choice([1, 2, 3, 7, 64, 129, 300, 1000, 2500, 5000]))
        B = max(1, min(B, 10000 // T))
        out.append((B, T, d, K, D_h, int(rng.choice(FLAG_SETS))))
    return out


@pytest.mark.parametrize("B,T,d,K,D_h,flags", _layer_shapes(2024, 16))
def test_random_layer_forward_backward(B, T, d, K, D_h, flags):
    _check_bf16_backward(*_bf16_backward_case(B, T, d, K, D_h, seed=B * 131 + T + d + K,
                                              flags=flags))
    assert eg.engram_get_status() == 0


def _decode_shapes(seed, n):
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(1, 300)), int(rng.integers(2, 9)), int(rng.choice([256, 512])),
             int(rng.integers(1, 5)), int(rng.choice([32, 64, 128])),
             int(rng.choice([0, eg.CONV_DILATED, eg.NORM_SCALES, eg.CONV_PRENORM])))
            for _ in range(n)]


@pytest.mark.parametrize("B,T,d,K,D_h,flags", _decode_shapes(77, 8))
def test_random_decode_streaming(B, T, d, K, D_h, flags):
    r = np.random.default_rng(B * 7 + T + d)
    E = 2 * K * D_h
    rows = synth.primes_at_most(1009, 2 * K)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, np.ones((2 * K, 3), np.uint64),
                      flags=flags)
    e = r.standard_normal((B, T, E)).astype(np.float32)
    h = r.standard_normal((B, T, 1, d)).astype(np.float32)
    Wk = (r.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (r.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    n_par = eg.engram_param_floats(cfg)
    block = (r.standard_normal(n_par) * 0.5).astype(np.float32)
    if n_par > 4 * d:  # learnable scales near 1
        block[4 * d:] = (1.0 + 0.3 * r.standard_normal(n_par - 4 * d)).astype(np.float32)
    f64, b = O.bf16_bits_to_f64, synth.to_bf16_bits
    ref = O.layer_forward_v(f64(b(e)).reshape(B * T, E), f64(b(h)).reshape(B * T, 1, d),
                            f64(b(Wk)), f64(b(Wv)), block, T, flags)["out"].reshape(B, T, 1, d)
    state = torch.zeros((B, 1, 3 * O.dilation_of(flags), d), device="cuda")
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, B)
    w = ws(fb)
    Wk_d, Wv_d, blk = bf16_dev(Wk), bf16_dev(Wv), dev(block)
    out = torch.empty((B, 1, 1, d), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        eg.engram_forward(cfg, None, None, bf16_dev(np.ascontiguousarray(e[:, t])),
                          bf16_dev(np.ascontiguousarray(h[:, t])), Wk_d, Wv_d, blk, state, out,
                          None, B, 1, w, fb)
        assert max_rel_err(out[:, 0].float().cpu().numpy(), ref[:, t]) <= 2e-2, t
    assert eg.engram_get_status() == 0
