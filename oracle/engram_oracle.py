"""CPU oracle of the Engram conditional-memory layer (plain, slow, fp64).

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only
the tests, the smoke check in ``__graft_entry__`` and the ``cpu_baseline`` /
reference arm of ``bench.py`` may call it.  It shares no code with the CUDA
path: every step below is written out from its definition.

Sources (the pages are secondary write-ups of "Conditional Memory via Scalable
Lookup: A New Axis of Sparsity for Large Language Models"):

* [p1] reportify.cn, tag page 条件记忆 -- bullet digests: 技术架构与原理,
  技术方案 (tokenizer compression, multi-head hashing), 关键技术.
* [p2] sechub.in, Q&A answer -- 2-gram / 3-gram suffixes, context-aware gate,
  short depthwise causal conv.
* [p4] gitcode.csdn.net, "Engram 到底怎么工作的" -- the four steps (第一步 ..
  第四步) and end-to-end training with consistent slot gradients.
* [p5] discuss.deepseek.club, section 二.1 (1) sparse hash retrieval,
  二.1 (2) context-aware gate and 1-D conv, 二.2 multi-branch integration.

Choices the pages leave open are fixed as follows (each one is a reading,
listed with the others in the design notes of the repository):

* vocabulary projection: compressed id = rank of the raw id's key among the
  distinct keys, ordered by first occurrence in ascending raw id.
* positions before the start of a sequence hold the PAD id = V_c.
* hash head j (order n = 2 for j < K, 3 otherwise) of the suffix n-gram
  g = (c_t, c_{t-1}, c_{t-2}): x = XOR_i (g_i * mult[j, i]) in wrap-around
  64-bit arithmetic, slot = x mod P_j (P_j prime).
* e_t concatenates the J head rows in head order (2-gram heads first).
* k = W_k e, v = W_v e with W stored [d, E] (no bias); RMSNorm without a
  learnable scale, eps 1e-6; alpha = sigmoid(<RMSNorm(h), RMSNorm(k)> / sqrt(d)).
* y_t = sum_{i=0..3} w[:, i] * vt_{t-3+i} (depthwise, dilation 1, zero before
  the sequence start); out = h + vt + SiLU(y) with vt = alpha * v.
* M branches: own W_k and alpha each, shared table, W_v and conv weights.
* sparse table gradient: per touched row, the sum of the de segments of the
  tokens that hit it, in ascending flat token order.

Parity pins: the test-suite checks every function here against closed forms,
invariants, hand-worked cases and finite differences (see tests/test_oracle_*).
"""
from __future__ import annotations

import math

import numpy as np

RMS_EPS = 1e-6
CONV_K = 4


# ----------------------------------------------------------------------------
# bf16 storage helpers (the oracle's own, round-to-nearest-even)
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 (exact)."""
    u32 = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns, one rounding, to nearest, ties to even.

    Written from the definition: among the two bf16 neighbours of x pick the
    nearer, on a tie the one whose last mantissa bit is 0.  Finite inputs only.
    """
    x = np.asarray(x, dtype=np.float64)
    # bf16 has 8 significant bits; spacing at x is 2^(floor(log2|x|) - 7)
    ax = np.abs(x)
    out = np.zeros(x.shape, dtype=np.float64)
    nz = ax > 0
    _, e2 = np.frexp(ax[nz])             # ax = m * 2^e2, m in [0.5, 1): exact exponent
    ex = e2.astype(np.float64) - 1.0     # ax in [2^ex, 2^(ex+1))
    ex = np.maximum(ex, -126.0)          # subnormal range keeps the spacing of 2^-133
    ulp = np.exp2(ex - 7.0)
    q = ax[nz] / ulp                     # exact in fp64 (power-of-two scaling)
    lo = np.floor(q)
    frac = q - lo
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(lo, 2.0) == 1.0))
    out[nz] = (lo + up) * ulp
    out = np.copysign(out, x)
    f32 = out.astype(np.float32)         # exact: out is representable in bf16
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------
# retrieval: [p5 二.1 (1)], [p4 第一步/第二步], [p1 技术方案]
# ----------------------------------------------------------------------------

def build_vocab_proj(keys: np.ndarray):
    """Vocabulary projection ([p5 二.1 (1)] 词汇投影; [p1] 分词器压缩).

    Raw ids that share a canonical key map to one compressed id.  Compressed
    ids number the distinct keys in order of first occurrence by raw id.
    Returns (proj int32 [V], V_c).
    """
    first = {}
    proj = np.empty(len(keys), dtype=np.int32)
    for raw_id, key in enumerate(np.asarray(keys).tolist()):
        if key not in first:
            first[key] = len(first)
        proj[raw_id] = first[key]
    return proj, len(first)


def compress(proj: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """c = proj[x]; a raw id outside [0, V) is an error."""
    ids = np.asarray(ids)
    if ids.size and (ids.min() < 0 or ids.max() >= len(proj)):
        raise ValueError("raw token id out of range")
    return proj[ids].astype(np.int64)


def suffix_ngrams(c: np.ndarray, pad: int) -> np.ndarray:
    """Suffix n-grams of every position ([p4 第一步]: the last two and the last
    three tokens; [p2]: 2-gram and 3-gram suffixes).

    c: [B, T] compressed ids.  Returns g [B, T, 3] with g[..., i] = c_{t-i},
    and PAD wherever t - i < 0 inside the sequence.
    """
    B, T = c.shape
    g = np.full((B, T, 3), pad, dtype=np.int64)
    for i in range(3):
        if T > i:
            g[:, i:, i] = c[:, : T - i]
    return g


def hash_heads(g: np.ndarray, mult: np.ndarray, rows: np.ndarray, K: int) -> np.ndarray:
    """Multi-head hashing ([p5 二.1 (1)] 多头哈希; [p4 第二步]).

    Head j < K hashes the 2-gram (g_0, g_1), head j >= K the 3-gram
    (g_0, g_1, g_2): x = XOR over positions of g_i * mult[j, i] (mod 2^64),
    slot = x mod P_j.  g: [..., 3] int64; returns int32 [..., 2K].
    """
    J = 2 * K
    g64 = np.asarray(g, dtype=np.int64).astype(np.uint64)
    out = np.empty(g.shape[:-1] + (J,), dtype=np.int32)
    for j in range(J):
        order = 2 if j < K else 3
        x = np.zeros(g.shape[:-1], dtype=np.uint64)
        for i in range(order):
            x ^= g64[..., i] * np.uint64(mult[j, i])      # numpy uint64 wraps mod 2^64
        out[..., j] = (x % np.uint64(rows[j])).astype(np.int32)
    return out


def hash_indices(proj, ids, mult, rows, K, V_c):
    """Steps 1-3 for a batch of sequences: ids [B, T] -> idx [B, T, 2K]."""
    c = compress(proj, ids)
    return hash_heads(suffix_ngrams(c, V_c), mult, rows, K)


def hash_indices_decode(proj, ids_step, state, mult, rows, K):
    """One decode step: ids_step [B] raw ids, state [B, 2] = (c_{t-1}, c_{t-2}).

    Returns (idx [B, 2K], new_state)."""
    c = compress(proj, ids_step)
    g = np.stack([c, state[:, 0].astype(np.int64), state[:, 1].astype(np.int64)], axis=-1)
    idx = hash_heads(g, mult, rows, K)
    new_state = np.stack([c, state[:, 0]], axis=-1).astype(np.int32)
    return idx, new_state


def gather(idx: np.ndarray, tables) -> np.ndarray:
    """e_t = concatenation over heads j of T_j[idx_j] ([p5 二.1 (1)] 拼接检索结果).

    tables: list of J arrays [P_j, D_h].  idx: [..., J].  Returns [..., J*D_h]
    in the tables' dtype (an exact copy).  A slot of -1 (a token whose n-gram
    holds an invalid id) reads no row: its D_h entries are zero."""
    parts = []
    for j in range(len(tables)):
        t = np.asarray(tables[j])
        ij = idx[..., j]
        part = t[np.where(ij >= 0, ij, 0)]
        part[ij < 0] = 0
        parts.append(part)
    return np.concatenate(parts, axis=-1)


def hot_rows(idx: np.ndarray, rows, C: int):
    """The C packed-table rows that a sample of hash indices addresses most
    often: the rows a GPU-memory cache in front of a host-memory table keeps
    ([p1] 系统效率优化 / [p2] 多级缓存设计: by the Zipfian frequencies of
    n-grams, frequent rows near the GPU, the long tail further away).

    idx [..., J]; rows = P_j.  Head j's slot s is packed row
    P_0 + .. + P_{j-1} + s; slots outside [0, P_j) address no row.  Rows are
    ranked by how many (token, head) pairs address them, ties by ascending
    row id.  Returns (top: int64 [C], the ranked rows then -1, n_out =
    min(C, distinct rows))."""
    rows = np.asarray(rows, dtype=np.int64)
    J = rows.size
    idx = np.asarray(idx, dtype=np.int64).reshape(-1, J)
    base = np.concatenate([[0], np.cumsum(rows)[:-1]])
    valid = (idx >= 0) & (idx < rows[None, :])
    packed = (base[None, :] + idx)[valid]
    uniq, counts = np.unique(packed, return_counts=True)
    order = np.lexsort((uniq, -counts))  # by count descending, then row ascending
    top = uniq[order][:C]
    out = np.full(C, -1, dtype=np.int64)
    out[: top.size] = top
    return out, int(top.size)


# ----------------------------------------------------------------------------
# fusion: [p5 二.1 (2)], [p4 第三步/第四步], [p2]
# ----------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis, no learnable scale."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    return z * sigmoid(z)


def causal_conv(vt: np.ndarray, w: np.ndarray, T: int) -> np.ndarray:
    """Depthwise causal conv of width 4 ([p2] short depthwise causal conv;
    [p5 二.1 (2)] 一维卷积).  vt: [N, M, d] in flat token order (N = B*T),
    w: [d, 4].  y_t = sum_i w[:, i] * vt_{t-3+i}, zero across sequence starts."""
    N = vt.shape[0]
    pos = np.arange(N) % T
    y = np.zeros_like(vt)
    for i in range(CONV_K):
        lag = CONV_K - 1 - i
        src = np.arange(N) - lag
        ok = pos >= lag
        y[ok] += w[None, :, i] * vt[src[ok]]
    return y


def layer_forward(e, h, Wk, Wv, conv_w, T):
    """Gate, value, conv and residual of one Engram layer, in fp64.

    e [N, E]; h [N, M, d]; Wk [M, d, E]; Wv [d, E]; conv_w [d, 4].
    Returns a dict with out [N, M, d] and the intermediates k, v, alpha, vt, y.
    """
    e = np.asarray(e, np.float64)
    h = np.asarray(h, np.float64)
    Wk = np.asarray(Wk, np.float64)
    Wv = np.asarray(Wv, np.float64)
    w = np.asarray(conv_w, np.float64)
    N, M, d = h.shape
    # key per branch and shared value ([p5 二.1 (2)]: h as query, e as key and value)
    k = np.stack([e @ Wk[m].T for m in range(M)], axis=1)          # [N, M, d]
    v = e @ Wv.T                                                    # [N, d]
    # context-aware gate ([p5 二.1 (2)] 门控因子; [p4 第三步])
    z = np.sum(rmsnorm(h) * rmsnorm(k), axis=-1) / math.sqrt(d)     # [N, M]
    alpha = sigmoid(z)
    vt = alpha[..., None] * v[:, None, :]                           # [N, M, d]
    y = causal_conv(vt, w, T)
    out = h + vt + silu(y)
    return dict(out=out, k=k, v=v, z=z, alpha=alpha, vt=vt, y=y)


def layer_forward_bf16(e_bits, h_bits, Wk_bits, Wv_bits, conv_w, T):
    """bf16 storage: inputs are bf16 bit patterns; the arithmetic is fp64 and
    the output is rounded to bf16 once."""
    r = layer_forward(bf16_bits_to_f64(e_bits), bf16_bits_to_f64(h_bits),
                      bf16_bits_to_f64(Wk_bits), bf16_bits_to_f64(Wv_bits), conv_w, T)
    r["out_bits"] = f64_to_bf16_bits(r["out"])
    return r


def decode_step(e, h, Wk, Wv, conv_w, conv_state):
    """One token per sequence.  e [B, E]; h [B, M, d]; conv_state [B, M, 3, d]
    holds vt of the three previous steps (oldest first, zeros at the start).
    Returns (out [B, M, d], alpha [B, M], new_state)."""
    e = np.asarray(e, np.float64)
    h = np.asarray(h, np.float64)
    Wk = np.asarray(Wk, np.float64)
    Wv = np.asarray(Wv, np.float64)
    w = np.asarray(conv_w, np.float64)
    st = np.asarray(conv_state, np.float64)
    B, M, d = h.shape
    k = np.stack([e @ Wk[m].T for m in range(M)], axis=1)
    v = e @ Wv.T
    alpha = sigmoid(np.sum(rmsnorm(h) * rmsnorm(k), axis=-1) / math.sqrt(d))
    vt = alpha[..., None] * v[:, None, :]
    y = w[None, None, :, 3] * vt
    for i in range(3):
        y = y + w[None, None, :, i] * st[:, :, i, :]
    out = h + vt + silu(y)
    new_state = np.concatenate([st[:, :, 1:, :], vt[:, :, None, :]], axis=2)
    return out, alpha, new_state


# ----------------------------------------------------------------------------
# backward ([p4]: end-to-end training, consistent gradients to the same slots)
# ----------------------------------------------------------------------------

def rmsnorm_backward(x, dxh, eps: float = RMS_EPS):
    """Gradient through xh = x * r, r = (mean(x^2) + eps)^(-1/2):
    dx = r*dxh - r^3 * x * <dxh, x> / d."""
    d = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return r * dxh - (r ** 3) * x * np.sum(dxh * x, axis=-1, keepdims=True) / d


def layer_backward(e, h, Wk, Wv, conv_w, T, dout, fwd=None):
    """All gradients of L = sum(dout * out) for one Engram layer, fp64.

    Returns dict: dh [N,M,d], dWk [M,d,E], dWv [d,E], dconv_w [d,4], de [N,E].
    """
    e = np.asarray(e, np.float64)
    h = np.asarray(h, np.float64)
    Wk = np.asarray(Wk, np.float64)
    Wv = np.asarray(Wv, np.float64)
    w = np.asarray(conv_w, np.float64)
    u = np.asarray(dout, np.float64)
    if fwd is None:
        fwd = layer_forward(e, h, Wk, Wv, w, T)
    k, v, alpha, vt, y = fwd["k"], fwd["v"], fwd["alpha"], fwd["vt"], fwd["y"]
    N, M, d = h.shape
    pos = np.arange(N) % T

    # out = h + vt + SiLU(y)
    sy = sigmoid(y)
    dy = u * sy * (1.0 + y * (1.0 - sy))
    dvt = u.copy()
    dconv_w = np.zeros((d, CONV_K))
    for i in range(CONV_K):
        lag = CONV_K - 1 - i
        tgt = np.arange(N) + lag               # y_{t+lag} reads vt_t through tap i
        ok = (pos + lag) < T
        dvt[ok] += w[None, :, i] * dy[tgt[ok]]
        src = np.arange(N) - lag
        ok2 = pos >= lag
        dconv_w[:, i] = np.sum(dy[ok2] * vt[src[ok2]], axis=(0, 1))

    # vt = alpha * v
    dalpha = np.sum(dvt * v[:, None, :], axis=-1)                   # [N, M]
    dv = np.sum(alpha[..., None] * dvt, axis=1)                     # [N, d]
    dz = dalpha * alpha * (1.0 - alpha)
    hh = rmsnorm(h)
    kh = rmsnorm(k)
    dhh = dz[..., None] * kh / math.sqrt(d)
    dkh = dz[..., None] * hh / math.sqrt(d)
    dh = u + rmsnorm_backward(h, dhh)
    dk = rmsnorm_backward(k, dkh)                                   # [N, M, d]

    dWk = np.stack([dk[:, m, :].T @ e for m in range(M)], axis=0)   # [M, d, E]
    dWv = dv.T @ e                                                  # [d, E]
    de = dv @ Wv
    for m in range(M):
        de = de + dk[:, m, :] @ Wk[m]
    return dict(dh=dh, dWk=dWk, dWv=dWv, dconv_w=dconv_w, de=de, dk=dk, dv=dv)


# ----------------------------------------------------------------------------
# formulation variants: the pages fix neither the conv's dilation, nor a norm
# before it, nor whether branches share it, nor learnable norm scales
# ([p2]: short depthwise causal conv; [p5 二.1 (2)] 一维卷积增强 then the
# residual; [p5 二.2] branches share table and W_v).  Each is a flag; with no
# flag the layer is the one above.
# ----------------------------------------------------------------------------

CONV_DILATED = 2      # taps at t, t-3, t-6, t-9 (dilation = the largest n-gram order)
CONV_PRENORM = 4      # the conv reads RMSNorm(vt) (times g_v with NORM_SCALES)
CONV_PER_BRANCH = 8   # conv weights per branch: [M, d, 4]
NORM_SCALES = 16      # learnable RMSNorm scales g_h, g_k (and g_v with CONV_PRENORM)


def param_count(flags: int, M: int, d: int) -> int:
    """Floats of the small-parameter block: conv weights ([M or 1] x d x 4),
    then with NORM_SCALES g_h [M, d], g_k [M, d] and, with CONV_PRENORM,
    g_v [M, d]."""
    n = (M if flags & CONV_PER_BRANCH else 1) * d * CONV_K
    if flags & NORM_SCALES:
        n += (3 if flags & CONV_PRENORM else 2) * M * d
    return n


def unpack_params(block, flags: int, M: int, d: int) -> dict:
    """The block's parts as fp64 arrays: w [M, d, 4] (a shared conv repeated
    over branches), g_h, g_k, g_v [M, d] (ones where absent)."""
    b = np.asarray(block, np.float64).reshape(-1)
    assert b.size == param_count(flags, M, d)
    Mc = M if flags & CONV_PER_BRANCH else 1
    w = b[: Mc * d * CONV_K].reshape(Mc, d, CONV_K)
    if Mc == 1:
        w = np.repeat(w, M, axis=0)
    off = Mc * d * CONV_K
    ones = np.ones((M, d))
    g_h = g_k = g_v = ones
    if flags & NORM_SCALES:
        g_h = b[off: off + M * d].reshape(M, d)
        g_k = b[off + M * d: off + 2 * M * d].reshape(M, d)
        if flags & CONV_PRENORM:
            g_v = b[off + 2 * M * d: off + 3 * M * d].reshape(M, d)
    return dict(w=w, g_h=g_h, g_k=g_k, g_v=g_v, Mc=Mc)


def dilation_of(flags: int) -> int:
    return 3 if flags & CONV_DILATED else 1


def causal_conv_v(c: np.ndarray, w: np.ndarray, T: int, dil: int) -> np.ndarray:
    """y_t = sum_i w[m, :, i] * c_{t-(3-i)*dil} per branch m, zero across
    sequence starts.  c: [N, M, d]; w: [M, d, 4]."""
    N = c.shape[0]
    pos = np.arange(N) % T
    y = np.zeros_like(c)
    for i in range(CONV_K):
        lag = (CONV_K - 1 - i) * dil
        src = np.arange(N) - lag
        ok = pos >= lag
        y[ok] += w[None, :, :, i] * c[src[ok]]
    return y


def layer_forward_v(e, h, Wk, Wv, block, T, flags):
    """The layer with the formulation variants of `flags`, fp64.

    z = <RMSNorm(h) g_h, RMSNorm(k) g_k> / sqrt(d), alpha = sigmoid(z),
    vt = alpha v, c = RMSNorm(vt) g_v with CONV_PRENORM else vt,
    y_t = sum_i w_i c_{t-(3-i) dil}, out = h + vt + SiLU(y)."""
    e = np.asarray(e, np.float64)
    h = np.asarray(h, np.float64)
    Wk = np.asarray(Wk, np.float64)
    Wv = np.asarray(Wv, np.float64)
    N, M, d = h.shape
    P = unpack_params(block, flags, M, d)
    k = np.stack([e @ Wk[m].T for m in range(M)], axis=1)
    v = e @ Wv.T
    z = np.sum(rmsnorm(h) * P["g_h"][None] * rmsnorm(k) * P["g_k"][None], axis=-1) / math.sqrt(d)
    alpha = sigmoid(z)
    vt = alpha[..., None] * v[:, None, :]
    c = rmsnorm(vt) * P["g_v"][None] if flags & CONV_PRENORM else vt
    y = causal_conv_v(c, P["w"], T, dilation_of(flags))
    out = h + vt + silu(y)
    return dict(out=out, k=k, v=v, z=z, alpha=alpha, vt=vt, c=c, y=y)


def decode_step_v(e, h, Wk, Wv, block, conv_state, flags):
    """One token per sequence with the variants of `flags`.  conv_state
    [B, M, 3 dil, d] holds the conv inputs c of the 3 dil previous steps,
    oldest first (zeros at the start).  Returns (out, alpha, new_state)."""
    e = np.asarray(e, np.float64)
    h = np.asarray(h, np.float64)
    Wk = np.asarray(Wk, np.float64)
    Wv = np.asarray(Wv, np.float64)
    st = np.asarray(conv_state, np.float64)
    B, M, d = h.shape
    dil = dilation_of(flags)
    P = unpack_params(block, flags, M, d)
    k = np.stack([e @ Wk[m].T for m in range(M)], axis=1)
    v = e @ Wv.T
    z = np.sum(rmsnorm(h) * P["g_h"][None] * rmsnorm(k) * P["g_k"][None], axis=-1) / math.sqrt(d)
    alpha = sigmoid(z)
    vt = alpha[..., None] * v[:, None, :]
    c = rmsnorm(vt) * P["g_v"][None] if flags & CONV_PRENORM else vt
    w = P["w"]
    y = w[None, :, :, 3] * c
    for i in range(3):
        lag = (3 - i) * dil                  # state index 3 dil - lag
        y = y + w[None, :, :, i] * st[:, :, 3 * dil - lag, :]
    out = h + vt + silu(y)
    new_state = np.concatenate([st[:, :, 1:, :], c[:, :, None, :]], axis=2)
    return out, alpha, new_state


def layer_backward_v(e, h, Wk, Wv, block, T, dout, flags):
    """All gradients of L = sum(dout * out) for the variant layer, fp64:
    dh, dWk, dWv, de and dblock (the small-parameter block's gradient, in
    the block's layout)."""
    e = np.asarray(e, np.float64)
    h = np.asarray(h, np.float64)
    Wk = np.asarray(Wk, np.float64)
    Wv = np.asarray(Wv, np.float64)
    u = np.asarray(dout, np.float64)
    N, M, d = h.shape
    P = unpack_params(block, flags, M, d)
    f = layer_forward_v(e, h, Wk, Wv, block, T, flags)
    k, v, alpha, vt, c, y = f["k"], f["v"], f["alpha"], f["vt"], f["c"], f["y"]
    w, dil = P["w"], dilation_of(flags)
    pos = np.arange(N) % T
    sy = sigmoid(y)
    dy = u * sy * (1.0 + y * (1.0 - sy))
    dc = np.zeros_like(c)
    dw = np.zeros((M, d, CONV_K))
    for i in range(CONV_K):
        lag = (CONV_K - 1 - i) * dil
        tgt = np.arange(N) + lag               # y_{t+lag} reads c_t through tap i
        ok = (pos + lag) < T
        dc[ok] += w[None, :, :, i] * dy[tgt[ok]]
        src = np.arange(N) - lag
        ok2 = pos >= lag
        dw[:, :, i] = np.sum(dy[ok2] * c[src[ok2]], axis=0)
    dg_v = np.zeros((M, d))
    if flags & CONV_PRENORM:
        ch = rmsnorm(vt)
        dg_v = np.sum(dc * ch, axis=0)
        dvt = u + rmsnorm_backward(vt, dc * P["g_v"][None])
    else:
        dvt = u + dc
    dalpha = np.sum(dvt * v[:, None, :], axis=-1)
    dv = np.sum(alpha[..., None] * dvt, axis=1)
    dz = dalpha * alpha * (1.0 - alpha)
    hh, kh = rmsnorm(h), rmsnorm(k)
    gh, gk = P["g_h"][None], P["g_k"][None]
    dhh = dz[..., None] * gh * gk * kh / math.sqrt(d)
    dkh = dz[..., None] * gh * gk * hh / math.sqrt(d)
    dg_h = np.sum(dz[..., None] * hh * kh * gk, axis=0) / math.sqrt(d)
    dg_k = np.sum(dz[..., None] * hh * kh * gh, axis=0) / math.sqrt(d)
    dh = u + rmsnorm_backward(h, dhh)
    dk = rmsnorm_backward(k, dkh)
    dWk = np.stack([dk[:, m, :].T @ e for m in range(M)], axis=0)
    dWv = dv.T @ e
    de = dv @ Wv
    for m in range(M):
        de = de + dk[:, m, :] @ Wk[m]
    parts = [(dw if P["Mc"] == M else dw.sum(axis=0, keepdims=True)).reshape(-1)]
    if flags & NORM_SCALES:
        parts += [dg_h.reshape(-1), dg_k.reshape(-1)]
        if flags & CONV_PRENORM:
            parts.append(dg_v.reshape(-1))
    return dict(dh=dh, dWk=dWk, dWv=dWv, de=de, dblock=np.concatenate(parts), dk=dk, dv=dv)


def table_grad_f64(idx, de, rows, D_h):
    """Dense fp64 table gradient: dT_j[s] = sum of de_t[j-th segment] over the
    tokens t with idx[t, j] = s.  Returns a list of J arrays [P_j, D_h]."""
    idx = np.asarray(idx).reshape(-1, len(rows))
    de = np.asarray(de, np.float64).reshape(idx.shape[0], -1)
    out = []
    for j, P in enumerate(rows):
        g = np.zeros((int(P), D_h))
        np.add.at(g, idx[:, j], de[:, j * D_h:(j + 1) * D_h])
        out.append(g)
    return out


def table_grad_segments(idx, de, rows, D_h):
    """Sparse table gradient in fp32, as the deterministic reduction defines it.

    Keys are packed-table row ids (head j's slot s is row sum_{i<j} P_i + s),
    ascending and unique.  Each row's gradient is the fp32 sum, started from
    +0, of its tokens' de segments taken one by one in ascending flat token
    order.  Returns (keys int64 [U], grads float32 [U, D_h]).
    """
    idx = np.asarray(idx).reshape(-1, len(rows)).astype(np.int64)
    de = np.asarray(de, np.float32).reshape(idx.shape[0], -1)
    N, J = idx.shape
    base = np.concatenate([[0], np.cumsum(np.asarray(rows, np.int64))[:-1]])
    sums = {}
    for t in range(N):                      # ascending flat token order
        for j in range(J):
            key = int(base[j] + idx[t, j])
            seg = de[t, j * D_h:(j + 1) * D_h]
            if key not in sums:
                sums[key] = np.zeros(D_h, dtype=np.float32)
            sums[key] = (sums[key] + seg).astype(np.float32)   # one fp32 add per element
    keys = np.array(sorted(sums), dtype=np.int64)
    grads = np.stack([sums[k] for k in keys.tolist()]) if len(keys) else np.zeros((0, D_h), np.float32)
    return keys, grads.astype(np.float32)


def table_grad_segments_fast(idx, de, rows, D_h):
    """The same reduction as `table_grad_segments`, vectorised across rows for
    larger cases: tokens of each row are visited in ascending order and added
    one at a time in fp32."""
    idx = np.asarray(idx).reshape(-1, len(rows)).astype(np.int64)
    de = np.asarray(de, np.float32).reshape(idx.shape[0], -1)
    N, J = idx.shape
    base = np.concatenate([[0], np.cumsum(np.asarray(rows, np.int64))[:-1]])
    key = (base[None, :] + idx).reshape(-1)                       # item (t, j) -> row id
    tok = np.repeat(np.arange(N), J)
    head = np.tile(np.arange(J), N)
    order = np.lexsort((tok, key))                                # by row id, then token
    key_s, tok_s, head_s = key[order], tok[order], head[order]
    if key_s.size == 0:
        return np.zeros(0, np.int64), np.zeros((0, D_h), np.float32)
    starts = np.flatnonzero(np.r_[True, key_s[1:] != key_s[:-1]])
    lens = np.diff(np.r_[starts, key_s.size])
    U = starts.size
    acc = np.zeros((U, D_h), dtype=np.float32)
    for step in range(int(lens.max())):
        live = lens > step
        p = starts[live] + step
        seg = de[tok_s[p][:, None], head_s[p][:, None] * D_h + np.arange(D_h)[None, :]]
        acc[live] = (acc[live] + seg).astype(np.float32)
    return key_s[starts], acc
