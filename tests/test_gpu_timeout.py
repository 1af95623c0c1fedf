"""The bounded device-side waits give up and wind down instead of hanging.

With the test-only flag ENGRAM_TEST_STALL a bf16 call's tensor-core kernels
get no second operand (and the backward's row kernel no copies), so their
first wait cannot complete, and every wait of the call is limited to about
1 ms.  The call must return, the status word must report
ENGRAM_STATUS_TIMEOUT, and the device must stay usable: the same layer
without the flag then matches the oracle.  Nothing here traps or faults:
the kernels give up, let what they issued land, free their tensor memory
and return normally.
"""
import time

import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O
from tests.engram_cases import Layer, bf16_bits, bf16_dev, dev, max_rel_err, packed_table
from tests.test_gpu_backward import _check_bf16_backward

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
STALL = eg.TEST_STALL


def _unit_layer(B, T, d, K, D_h, seed, flags=0):
    """A unit-scale bf16 layer (tables N(0,1), W N(0,1/E)) and its inputs."""
    rng = np.random.default_rng(seed)
    J, E, N = 2 * K, 2 * K * D_h, B * T
    rows = synth.primes_at_most(2003, J)
    tables = [rng.standard_normal((P, D_h)).astype(np.float32) for P in rows]
    Wk = (rng.standard_normal((1, d, E)) / np.sqrt(E)).astype(np.float32)
    Wv = (rng.standard_normal((d, E)) / np.sqrt(E)).astype(np.float32)
    h = rng.standard_normal((B, T, 1, d)).astype(np.float32)
    conv_w = (rng.standard_normal((d, 4)) * 0.5).astype(np.float32)
    idx = np.stack([rng.integers(0, P, N) for P in rows], -1).astype(np.int32)
    mult = np.ones((J, 3), np.uint64)
    cfg = eg.make_cfg(K, D_h, d, 1, 1000, 770, eg.BF16, rows, mult, flags=flags)
    L = Layer(cfg, B, T, packed_table(tables, "bf16"), bf16_dev(h), bf16_dev(Wk), bf16_dev(Wv),
              dev(conv_w), torch.bfloat16)
    return L, dict(rows=rows, tables=tables, Wk=Wk, Wv=Wv, h=h, conv_w=conv_w, idx=idx,
                   mult=mult, K=K, D_h=D_h, d=d, flags=flags)


def _stalled(L, p):
    """The same layer with ENGRAM_TEST_STALL set in its configuration."""
    L.cfg = eg.make_cfg(p["K"], p["D_h"], p["d"], 1, 1000, 770, eg.BF16, p["rows"], p["mult"],
                        flags=p["flags"] | STALL)
    return L


def _plain(L, p):
    L.cfg = eg.make_cfg(p["K"], p["D_h"], p["d"], 1, 1000, 770, eg.BF16, p["rows"], p["mult"],
                        flags=p["flags"])
    return L


@pytest.mark.parametrize("B,T,d", [
    (3, 100, 256),    # narrow tiles (pair tiles of 256 x 64)
    (2, 2500, 256),   # wide tiles (256 x 256)
])
def test_forward_wait_runs_out_then_next_call_is_correct(B, T, d):
    assert eg.engram_get_status() == 0
    L, p = _unit_layer(B, T, d, 2, 32, seed=B * 13 + T)
    N = B * T
    idx = dev(p["idx"].reshape(B, T, -1))
    L.forward(idx)                           # set-up of the kernels, untimed
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    t0 = time.perf_counter()
    _stalled(L, p).forward(idx)              # returns: the waits give up
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    st = eg.engram_get_status()              # reads and clears the status word
    assert st & eg.STATUS_TIMEOUT, st
    assert wall < 1.5, wall                  # ~1 ms limits, not the normal 2 s
    assert eg.engram_get_status() == 0
    # the device is usable: the same layer without the flag matches the oracle
    out = _plain(L, p).forward(idx)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    tb = [synth.to_bf16_bits(t) for t in p["tables"]]
    e_bits = O.gather(p["idx"], tb)
    ref = O.layer_forward_bf16(e_bits, synth.to_bf16_bits(p["h"]).reshape(N, 1, d),
                               synth.to_bf16_bits(p["Wk"]), synth.to_bf16_bits(p["Wv"]),
                               p["conv_w"], T)
    got = O.bf16_bits_to_f64(bf16_bits(out)).reshape(N, 1, d)
    assert max_rel_err(got, O.bf16_bits_to_f64(ref["out_bits"])) <= TOL_BF16


@pytest.mark.parametrize("B,T,d,flags", [
    (3, 100, 256, eg.SAVE_KV),   # the row kernel and the dW / de GEMMs
    (2, 700, 256, 0),            # also the [k | v] GEMM (k and v recomputed)
])
def test_backward_wait_runs_out_then_next_call_is_correct(B, T, d, flags):
    assert eg.engram_get_status() == 0
    L, p = _unit_layer(B, T, d, 2, 32, seed=B * 19 + T, flags=flags)
    N = B * T
    idx = dev(p["idx"].reshape(B, T, -1))
    rng = np.random.default_rng(B + T)
    dout = rng.standard_normal((N, 1, d)).astype(np.float32)
    L.forward(idx)
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    t0 = time.perf_counter()
    _stalled(L, p).backward(idx, dev(dout))
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    st = eg.engram_get_status()
    assert st & eg.STATUS_TIMEOUT, st
    assert wall < 1.5, wall
    assert eg.engram_get_status() == 0
    g = _plain(L, p).backward(idx, dev(dout))
    torch.cuda.synchronize()
    assert eg.engram_get_status() == 0
    f64 = O.bf16_bits_to_f64
    e_ref = f64(O.gather(p["idx"], [synth.to_bf16_bits(t) for t in p["tables"]]))
    ref = O.layer_backward(e_ref, f64(synth.to_bf16_bits(p["h"])).reshape(N, 1, d),
                           f64(synth.to_bf16_bits(p["Wk"])), f64(synth.to_bf16_bits(p["Wv"])),
                           p["conv_w"], T, dout)
    ref["e"] = e_ref
    ref["Wk_bf"] = f64(synth.to_bf16_bits(p["Wk"]))
    ref["Wv_bf"] = f64(synth.to_bf16_bits(p["Wv"]))
    _check_bf16_backward(g, ref, p["idx"], p["rows"], p["D_h"])
