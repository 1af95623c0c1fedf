"""Seeded synthetic inputs for the Engram layer.

This module only draws random numbers and fixes workload shapes.  It holds
none of the layer's arithmetic (no projection, hashing, gathering, gating or
convolution), so both the CPU oracle side and the CUDA side of the tests can
take their inputs from here without sharing any of the method's code.

Workloads (all synthetic: the pages' corpora, tokenizer and trained weights
are not available):

* ``tiny``       1 x 64 tokens, fp32, d 64, K 2 heads per order x 1,009 rows x 16
* ``layer27b``   8 x 4,096 tokens, bf16, d 2,560, K 8 x ~4.45M rows x 80 (5.7B params)
* ``train``      the tiny shapes with 4 branches, two Engram layers (2 and 6)
* ``decode``     256 sequences x 1 token per step, d 4,096, K 8 x ~6.35M rows x 128
* ``hosttable``  4 x 2,048 tokens, d 2,560, K 8 x ~39.06M rows x 160 in host memory

Token ids follow a Zipf(1.1) law over the raw vocabulary; the vocabulary
projection is stood in for by a random merge map that gives about 23% of the
raw ids the key of another id (the pages: tokenizer compression shrinks a
~128k vocabulary by about 23%).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

MASK64 = (1 << 64) - 1


# ----------------------------------------------------------------------------
# random streams
# ----------------------------------------------------------------------------

def splitmix64(seed: int, n: int) -> np.ndarray:
    """n outputs of the SplitMix64 generator (Steele, Lea & Flood, OOPSLA 2014).

    Used only to draw the hash multipliers, which are parameters of the hash
    family and are passed to both implementations as inputs.
    """
    out = np.empty(n, dtype=np.uint64)
    state = seed & MASK64
    for i in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        out[i] = z ^ (z >> 31)
    return out


def hash_multipliers(seed_layer: int, J: int) -> np.ndarray:
    """[J, 3] odd 64-bit multipliers, one per head and n-gram position."""
    return splitmix64(seed_layer, 3 * J).reshape(J, 3) | np.uint64(1)


def _is_prime(n: int) -> bool:
    if n < 2:
        return False
    if n % 2 == 0:
        return n == 2
    f = 3
    while f * f <= n:
        if n % f == 0:
            return False
        f += 2
    return True


def primes_at_most(x: int, count: int) -> List[int]:
    """The `count` largest primes <= x, in descending order."""
    out = []
    n = x
    while len(out) < count:
        if _is_prime(n):
            out.append(n)
        n -= 1
    return out


def zipf_ids(rng: np.random.Generator, V: int, s: float, n: int,
             perm: Optional[np.ndarray] = None) -> np.ndarray:
    """n raw token ids, rank r (1-based) drawn with p(r) ~ r^-s by inverse CDF,
    then sent through a random permutation of the vocabulary (drawn from rng
    after the ranks, unless `perm` gives it: more text of the same
    distribution)."""
    p = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    r = np.searchsorted(cdf, rng.random(n), side="right")
    r = np.minimum(r, V - 1)
    if perm is None:
        perm = rng.permutation(V)
    return perm[r].astype(np.int32)


def merge_keys(rng: np.random.Generator, V: int, V_c: int) -> np.ndarray:
    """int64 key per raw id: V_c random representatives get distinct random
    keys, every other id copies the key of a random representative."""
    reps = rng.choice(V, size=V_c, replace=False)
    keys_rep = rng.choice(1 << 62, size=V_c, replace=False).astype(np.int64)
    keys = np.empty(V, dtype=np.int64)
    keys[reps] = keys_rep
    others = np.setdiff1d(np.arange(V), reps)
    keys[others] = keys_rep[rng.integers(0, V_c, size=others.size)]
    return keys


def compressed_vocab(V: int, merge_frac: float = 0.23) -> int:
    return V - int(round(merge_frac * V))


# ----------------------------------------------------------------------------
# workload shapes
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    B: int
    T: int
    V: int
    K: int
    D_h: int
    d: int
    dtype: str                 # "f32" or "bf16"
    rows: List[int]            # P_j, one prime per head, J = 2K entries
    M: int = 1                 # hidden-state branches
    n_layers: int = 1
    steps: int = 1             # decode steps

    @property
    def J(self) -> int:
        return 2 * self.K

    @property
    def E(self) -> int:
        return self.J * self.D_h

    @property
    def N(self) -> int:
        return self.B * self.T

    @property
    def V_c(self) -> int:
        return compressed_vocab(self.V)

    def table_params(self) -> int:
        return sum(self.rows) * self.D_h


def workload(name: str) -> Workload:
    if name == "tiny":
        return Workload("tiny", 1, 1, 64, 1000, 2, 16, 64, "f32", [1009] * 4)
    if name == "layer27b":
        return Workload("layer27b", 2, 8, 4096, 129280, 8, 80, 2560, "bf16",
                        primes_at_most(4_450_001, 16))
    if name == "train":
        return Workload("train", 3, 1, 64, 1000, 2, 16, 64, "f32", [1009] * 4,
                        M=4, n_layers=2)
    if name == "decode":
        return Workload("decode", 4, 256, 1, 129280, 8, 128, 4096, "bf16",
                        primes_at_most(13_000_000_000 // (16 * 128), 16), steps=2000)
    if name == "hosttable":
        return Workload("hosttable", 5, 4, 2048, 129280, 8, 160, 2560, "bf16",
                        primes_at_most(39_062_500, 16))
    raise KeyError(name)


def custom(name: str, seed: int, B: int, T: int, V: int, K: int, D_h: int, d: int,
           dtype: str, rows: List[int], M: int = 1) -> Workload:
    assert len(rows) == 2 * K
    return Workload(name, seed, B, T, V, K, D_h, d, dtype, list(rows), M=M)


# ----------------------------------------------------------------------------
# host-side input sets (small workloads, numpy)
# ----------------------------------------------------------------------------

def layer_seed(w: Workload, layer: int) -> int:
    return w.seed * 1000 + layer


def host_inputs(w: Workload, layer: int = 0, ids: Optional[np.ndarray] = None) -> dict:
    """All inputs of one Engram layer as numpy arrays (fp32 values; bf16
    workloads round them to bf16 bit patterns with `to_bf16_bits`).

    The returned dict holds: ids [B,T] int32, keys [V] int64, mult [J,3] uint64,
    rows [J] int64, tables (list of J arrays [P_j, D_h]), h [B,T,M,d],
    Wk [M,d,E], Wv [d,E], conv_w [d,4], dout [B,T,M,d].
    """
    rng = np.random.default_rng(layer_seed(w, layer))
    base = np.random.default_rng(w.seed)
    if ids is None:
        ids = zipf_ids(base, w.V, 1.1, w.N).reshape(w.B, w.T)
    keys = merge_keys(np.random.default_rng(w.seed + 77), w.V, w.V_c)
    mult = hash_multipliers(layer_seed(w, layer), w.J)
    tables = [(rng.standard_normal((P, w.D_h)) * 0.02).astype(np.float32) for P in w.rows]
    h = rng.standard_normal((w.B, w.T, w.M, w.d)).astype(np.float32)
    Wk = (rng.standard_normal((w.M, w.d, w.E)) * 0.02).astype(np.float32)
    Wv = (rng.standard_normal((w.d, w.E)) * 0.02).astype(np.float32)
    conv_w = (rng.standard_normal((w.d, 4)) * 0.5).astype(np.float32)
    dout = rng.standard_normal((w.B, w.T, w.M, w.d)).astype(np.float32)
    return dict(ids=ids.astype(np.int32), keys=keys, mult=mult,
                rows=np.array(w.rows, dtype=np.int64), tables=tables, h=h, Wk=Wk,
                Wv=Wv, conv_w=conv_w, dout=dout)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even.  Used only to
    store generated fp32 draws at bf16 precision."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def seeded_floats(seed: int, shape, scale: float = 1.0) -> np.ndarray:
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


# ----------------------------------------------------------------------------
# device-side input sets (large bf16 workloads, torch on the GPU)
# ----------------------------------------------------------------------------

def device_table(w: Workload, layer: int = 0, device="cuda"):
    """The packed bf16 table [sum(P_j) * D_h], N(0, 0.02), drawn on the device
    from a seeded torch generator (tens of GB do not fit a host round trip)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(layer_seed(w, layer) * 7 + 1)
    n = w.table_params()
    t = torch.empty(n, dtype=torch.bfloat16, device=device)
    chunk = 1 << 30
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        t[s:e].normal_(0.0, 0.02, generator=g)
    return t


def device_dense(w: Workload, layer: int = 0, device="cuda"):
    """h [B,T,M,d], Wk [M,d,E], Wv [d,E] in bf16 and conv_w [d,4] fp32 on device."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(layer_seed(w, layer) * 7 + 2)
    h = torch.randn((w.B, w.T, w.M, w.d), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    Wk = (torch.randn((w.M, w.d, w.E), generator=g, device=device) * 0.02).to(torch.bfloat16)
    Wv = (torch.randn((w.d, w.E), generator=g, device=device) * 0.02).to(torch.bfloat16)
    conv_w = torch.randn((w.d, 4), generator=g, device=device) * 0.5
    return dict(h=h, Wk=Wk, Wv=Wv, conv_w=conv_w)


def host_ids_perm(w: Workload) -> np.ndarray:
    """The vocabulary permutation behind host_ids_keys(w)'s ids (its draws
    replayed), so that more ids of the same distribution can be drawn."""
    base = np.random.default_rng(w.seed)
    base.random(w.N * w.steps)
    return base.permutation(w.V)


def host_ids_keys(w: Workload):
    """ids [B*steps? , T] int32 and merge keys [V] int64 (numpy, host)."""
    base = np.random.default_rng(w.seed)
    n = w.N * w.steps
    ids = zipf_ids(base, w.V, 1.1, n)
    if w.steps > 1:
        ids = ids.reshape(w.steps, w.B)
    else:
        ids = ids.reshape(w.B, w.T)
    keys = merge_keys(np.random.default_rng(w.seed + 77), w.V, w.V_c)
    return ids.astype(np.int32), keys
