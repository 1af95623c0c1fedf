"""Shared helpers of the parity tests: device copies of the seeded inputs,
calls through the C ABI, and the comparison metric."""
from __future__ import annotations

import numpy as np
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth


def max_rel_err(a, b) -> float:
    """max_i |a_i - b_i| / max(|b_i|, 1e-3 * RMS(b)) -- the relative error with
    a floor, so entries near zero do not dominate."""
    a = np.asarray(a, np.float64).reshape(-1)
    b = np.asarray(b, np.float64).reshape(-1)
    if b.size == 0:
        return 0.0
    floor = 1e-3 * float(np.sqrt(np.mean(b * b))) + 1e-300
    return float(np.max(np.abs(a - b) / np.maximum(np.abs(b), floor)))


def dev(x, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t if dtype is None else t.to(dtype)


def bf16_dev(x_f32) -> torch.Tensor:
    bits = synth.to_bf16_bits(np.asarray(x_f32, np.float32))
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def cfg_of(w: synth.Workload, mult, V_c: int, M: int | None = None) -> eg.EngramCfg:
    return eg.make_cfg(w.K, w.D_h, w.d, w.M if M is None else M, w.V, V_c,
                       eg.F32 if w.dtype == "f32" else eg.BF16, w.rows, mult)


def ws(nbytes: int) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device="cuda")


def gpu_vocab_proj(keys: np.ndarray):
    V = keys.size
    k = dev(keys.astype(np.int64))
    proj = torch.empty(V, dtype=torch.int32, device="cuda")
    nb = eg.engram_workspace_size(None, eg.WS_VOCAB, V)
    w = ws(nb)
    V_c = eg.engram_build_vocab_proj(k, V, proj, w, nb)
    return proj, V_c


def gpu_hash(cfg, proj, ids: torch.Tensor, B: int, T: int, state=None) -> torch.Tensor:
    idx = torch.empty((B, T, cfg.J), dtype=torch.int32, device="cuda")
    eg.engram_hash_indices(cfg, proj, ids, B, T, state, idx)
    return idx


def packed_table(tables, dtype="f32") -> torch.Tensor:
    flat = np.concatenate([np.asarray(t, np.float32).reshape(-1) for t in tables])
    return dev(flat) if dtype == "f32" else bf16_dev(flat)


class Layer:
    """One Engram layer's device buffers for a forward (and backward) run."""

    def __init__(self, cfg, B, T, table, h, Wk, Wv, conv_w, dtype_t):
        self.cfg, self.B, self.T = cfg, B, T
        self.N = B * T
        self.table, self.h, self.Wk, self.Wv, self.conv_w = table, h, Wk, Wv, conv_w
        M, d, E = cfg.n_branch, cfg.d_model, cfg.E
        self.e = torch.empty((self.N, E), dtype=dtype_t, device="cuda")
        self.out = torch.empty((B, T, M, d), dtype=dtype_t, device="cuda")
        self.saved = ws(eg.engram_saved_size(cfg, self.N))
        self.fws_bytes = eg.engram_workspace_size(cfg, eg.WS_FORWARD, self.N)
        self.fws = ws(self.fws_bytes)

    def forward(self, idx, conv_state=None, table=True):
        eg.engram_forward(self.cfg, idx, self.table if table else None, self.e, self.h, self.Wk,
                          self.Wv, self.conv_w, conv_state, self.out, self.saved, self.B, self.T,
                          self.fws, self.fws_bytes)
        return self.out

    def backward(self, idx, dout):
        cfg, N, M, d, E = self.cfg, self.N, self.cfg.n_branch, self.cfg.d_model, self.cfg.E
        g = dict(
            dh=torch.empty((N, M, d), dtype=torch.float32, device="cuda"),
            dWk=torch.empty((M, d, E), dtype=torch.float32, device="cuda"),
            dWv=torch.empty((d, E), dtype=torch.float32, device="cuda"),
            # the small-parameter block's gradient: conv weights [d, 4], then
            # any learnable norm scales'
            dconv_w=torch.empty(eg.engram_param_floats(cfg), dtype=torch.float32,
                                device="cuda"),
            de=torch.empty((N, E), dtype=torch.float32, device="cuda"),
            keys=torch.empty(max(N * cfg.J, 1), dtype=torch.int64, device="cuda"),
            rows=torch.empty((max(N * cfg.J, 1), cfg.D_h), dtype=torch.float32, device="cuda"),
            n_unique=torch.zeros(1, dtype=torch.int32, device="cuda"),
        )
        nb = eg.engram_workspace_size(cfg, eg.WS_BACKWARD, N)
        w = ws(nb)
        eg.engram_backward(cfg, idx, self.e, self.h, self.Wk, self.Wv, self.conv_w, self.saved,
                           dout, g["dh"], g["dWk"], g["dWv"], g["dconv_w"], g["de"], g["keys"],
                           g["rows"], g["n_unique"], self.B, self.T, w, nb)
        return g
