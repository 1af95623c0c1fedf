"""Runs one kernel family of the library on seeded synthetic inputs of a given
shape, a few times, for profiling a kernel alone (e.g. under Nsight Compute)
without the rest of the layer's inputs on the device.

    python bench_cases.py fused \
        [--tokens 32768] [--d 2560] [--heads 16] [--dh 80] [--seq 4096] [--reps 3]
    python bench_cases.py gather [...]
    python bench_cases.py hash [...]
    python bench_cases.py decode \
        --tokens 256 --d 4096 --dh 128 --rows 1000003
    python bench_cases.py tablegrad [...]
    python bench_cases.py hostgather \
        --tokens 8192 --seq 2048 --dh 160 --rows 1000003
    python bench_cases.py backward [...]
    python bench_cases.py hostcache \
        --tokens 8192 --seq 2048 --dh 160 --rows 1000003 [--cache-rows 1048576]
    python bench_cases.py tiny [--reps 3]

`fused` runs engram_forward with table = NULL on random gathered rows, i.e.
the two tensor-core passes; `gather` gathers from a table of --rows rows per
head; `hash` runs the compress + n-gram + hash kernel; `decode` runs whole
decode steps (engram_decode_step: hash with the rolling n-gram state and
gather in one kernel, then one persistent launch for pass K, the gate and
pass V with the conv state) for --tokens
sequences of one token each;
`tiny` runs the tiny fp32 layer's step (hash, forward, backward; its own
fixed shape); `tablegrad` runs the sparse table gradient (sort by row, segment sums) on
fp32 rows of de for hash indices of Zipf(1.1) token ids; `hostgather` runs
engram_forward_hosttable on a table in pinned host memory; `backward` runs
the bf16 engram_backward (column walk, row kernel, GEMMs, sparse table
gradient) on random gathered rows, gates and output gradients; `hostcache`
runs engram_forward_hostcache with an HBM cache of the rows a second sample
of the same skewed (Zipf 1.2 per head) slot distribution addresses most.
Defaults are the
27B-shaped layer's dimensions.  Prints the device time per repetition.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["fused", "gather", "hash", "decode", "tablegrad",
                                       "hostgather", "backward", "hostcache", "tiny"])
    ap.add_argument("--tokens", type=int, default=32768)
    ap.add_argument("--seq", type=int, default=4096)
    ap.add_argument("--d", type=int, default=2560)
    ap.add_argument("--heads", type=int, default=16)
    ap.add_argument("--dh", type=int, default=80)
    ap.add_argument("--rows", type=int, default=4_450_001)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--cache-rows", type=int, default=1 << 20)
    ap.add_argument("--save-kv", action="store_true",
                    help="fused, backward: the forward keeps k and v for the backward")
    ap.add_argument("--dilated", action="store_true",
                    help="fused, backward, decode: the dilated conv (taps 3, 6, 9 tokens back)")
    ap.add_argument("--prenorm", action="store_true",
                    help="fused, backward, decode: the pre-conv RMSNorm (no learnable g_v)")
    a = ap.parse_args(argv)
    from hashed_gram_conditional_engram_b200 import build
    build.build()
    dev = torch.device("cuda")
    K = a.heads // 2
    E = a.heads * a.dh
    if a.kernel == "decode":
        a.seq = 1
    B = a.tokens // a.seq
    T = a.seq
    N = B * T
    rows = synth.primes_at_most(a.rows, a.heads)
    mult = synth.hash_multipliers(12345, a.heads)
    cfg = eg.make_cfg(K, a.dh, a.d, 1, 129280, synth.compressed_vocab(129280), eg.BF16, rows, mult,
                      flags=(eg.SAVE_KV if a.save_kv else 0) |
                      (eg.CONV_DILATED if a.dilated else 0) |
                      (eg.CONV_PRENORM if a.prenorm else 0))
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    if a.kernel == "tiny":
        run = _tiny_step(dev)
    elif a.kernel == "fused":
        e = (torch.randn((N, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        h = torch.randn((N, a.d), generator=g, device=dev).to(torch.bfloat16)
        Wk = (torch.randn((a.d, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        Wv = (torch.randn((a.d, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        cw = torch.randn((a.d, 4), generator=g, device=dev) * 0.5
        out = torch.empty_like(h)
        nb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        saved = torch.empty(eg.engram_saved_size(cfg, N), dtype=torch.uint8, device=dev)

        def run():
            eg.engram_forward(cfg, None, None, e, h, Wk, Wv, cw, None, out, saved, B, T, ws, nb)
    elif a.kernel == "backward":
        e = (torch.randn((N, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        h = torch.randn((N, a.d), generator=g, device=dev).to(torch.bfloat16)
        Wk = (torch.randn((a.d, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        Wv = (torch.randn((a.d, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        cw = torch.randn((a.d, 4), generator=g, device=dev) * 0.5
        saved = torch.empty(eg.engram_saved_size(cfg, N), dtype=torch.uint8, device=dev)
        saved[: N * 4].view(torch.float32).copy_(torch.rand((N,), generator=g, device=dev))
        if a.save_kv:  # k and v as a forward would have kept them
            off = (N * 4 + 255) // 256 * 256
            kv = saved[off: off + N * 2 * a.d * 4].view(torch.float32)
            kv.copy_((e.float() @ torch.cat([Wk, Wv]).float().T).reshape(-1))
        dout = torch.randn((N, a.d), generator=g, device=dev)
        rng = np.random.default_rng(3)
        idx = torch.from_numpy(np.stack([rng.integers(0, P, N) for P in rows], -1)
                               .astype(np.int32)).to(dev)
        dh = torch.empty((N, a.d), device=dev)
        dWk, dWv = torch.empty((a.d, E), device=dev), torch.empty((a.d, E), device=dev)
        dcw = torch.empty((a.d, 4), device=dev)
        keys_out = torch.empty(N * a.heads, dtype=torch.int64, device=dev)
        rows_out = torch.empty((N * a.heads, a.dh), device=dev)
        nu = torch.zeros(1, dtype=torch.int32, device=dev)
        nb = eg.engram_workspace_size(cfg, eg.WS_BACKWARD, N)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)

        def run():
            eg.engram_backward(cfg, idx, e, h, Wk, Wv, cw, saved, dout, dh, dWk, dWv, dcw, None,
                               keys_out, rows_out, nu, B, T, ws, nb)
    elif a.kernel == "gather":
        table = torch.empty(sum(rows) * a.dh, dtype=torch.bfloat16, device=dev)
        table.normal_(0.0, 0.02, generator=g)
        rng = np.random.default_rng(3)
        idx = torch.from_numpy(np.stack([rng.integers(0, P, N) for P in rows], -1)
                               .astype(np.int32)).to(dev)
        e = torch.empty((N, E), dtype=torch.bfloat16, device=dev)

        def run():
            eg.engram_gather(cfg, idx, table, N, e)
    elif a.kernel == "hostgather":
        n_el = sum(rows) * a.dh
        host = torch.empty(n_el, dtype=torch.bfloat16, pin_memory=True)
        buf = torch.empty(1 << 28, dtype=torch.bfloat16, device=dev)
        for lo in range(0, n_el, 1 << 28):
            hi = min(n_el, lo + (1 << 28))
            buf[: hi - lo].normal_(0.0, 0.02, generator=g)
            host[lo:hi].copy_(buf[: hi - lo])
        del buf
        rng = np.random.default_rng(3)
        idx = torch.from_numpy(np.stack([rng.integers(0, P, N) for P in rows], -1)
                               .astype(np.int32)).to(dev)
        e = torch.empty((N, E), dtype=torch.bfloat16, device=dev)
        side = torch.cuda.current_stream()

        def run():
            eg.engram_forward_hosttable(cfg, idx, host.data_ptr(), N, e, side, None)
    elif a.kernel == "hostcache":
        n_el = sum(rows) * a.dh
        host = torch.empty(n_el, dtype=torch.bfloat16, pin_memory=True)
        buf = torch.empty(1 << 28, dtype=torch.bfloat16, device=dev)
        for lo in range(0, n_el, 1 << 28):
            hi = min(n_el, lo + (1 << 28))
            buf[: hi - lo].normal_(0.0, 0.02, generator=g)
            host[lo:hi].copy_(buf[: hi - lo])
        del buf
        rng = np.random.default_rng(3)

        def skewed(n):
            return np.stack([(rng.zipf(1.2, n) - 1) % P for P in rows], -1).astype(np.int32)

        idx = torch.from_numpy(skewed(N)).to(dev)
        sample = torch.from_numpy(skewed(8 * N)).to(dev)
        C = a.cache_rows
        rb = eg.engram_workspace_size(cfg, eg.WS_HOSTCACHE_RANK, 8 * N)
        crow = torch.empty(C, dtype=torch.int64, device=dev)
        n_out = torch.zeros(1, dtype=torch.int32, device=dev)
        eg.engram_hostcache_rank(cfg, sample, 8 * N, C, crow, n_out,
                                 torch.empty(rb, dtype=torch.uint8, device=dev), rb)
        n_c = int(n_out.item())
        cache = torch.empty((max(n_c, 1), a.dh), dtype=torch.bfloat16, device=dev)
        cmap = torch.empty(eg.engram_table_rows(cfg), dtype=torch.int32, device=dev)
        eg.engram_hostcache_fill(cfg, host.data_ptr(), crow, n_c, cache, cmap)
        e = torch.empty((N, E), dtype=torch.bfloat16, device=dev)
        gb = eg.engram_workspace_size(cfg, eg.WS_HOSTCACHE_GATHER, N)
        gws = torch.empty(gb, dtype=torch.uint8, device=dev)
        n_miss = torch.zeros(1, dtype=torch.int32, device=dev)
        side = torch.cuda.current_stream()

        def run():
            eg.engram_forward_hostcache(cfg, idx, host.data_ptr(), cache, cmap, N, e, n_miss, gws,
                                        gb, side, None)
    elif a.kernel == "tablegrad":
        ids_np, keys_np = synth.host_ids_keys(synth.workload("layer27b"))
        keys = torch.from_numpy(keys_np).to(dev)
        proj = torch.empty(129280, dtype=torch.int32, device=dev)
        vb = eg.engram_workspace_size(None, eg.WS_VOCAB, 129280)
        eg.engram_build_vocab_proj(keys, 129280, proj, torch.empty(vb, dtype=torch.uint8, device=dev), vb)
        cfg32 = eg.make_cfg(K, a.dh, a.d, 1, 129280, synth.compressed_vocab(129280), eg.F32, rows,
                            mult)
        ids = torch.from_numpy(ids_np.reshape(-1)[:N].copy()).to(dev)
        idx = torch.empty((N, a.heads), dtype=torch.int32, device=dev)
        eg.engram_hash_indices(cfg32, proj, ids, B, T, None, idx)
        de = torch.randn((N, E), generator=g, device=dev)
        n_items = N * a.heads
        keys_out = torch.empty(n_items, dtype=torch.int64, device=dev)
        rows_out = torch.empty((n_items, a.dh), device=dev)
        nu = torch.zeros(1, dtype=torch.int32, device=dev)
        nb = eg.engram_workspace_size(cfg32, eg.WS_TABLE_GRAD, N)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)

        def run():
            eg.engram_table_grad(cfg32, idx, de, N, keys_out, rows_out, nu, ws, nb)
    elif a.kernel == "decode":
        table = torch.empty(sum(rows) * a.dh, dtype=torch.bfloat16, device=dev)
        table.normal_(0.0, 0.02, generator=g)
        h = torch.randn((N, a.d), generator=g, device=dev).to(torch.bfloat16)
        Wk = (torch.randn((a.d, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        Wv = (torch.randn((a.d, E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
        cw = torch.randn((a.d, 4), generator=g, device=dev) * 0.5
        out = torch.empty_like(h)
        e = torch.empty((N, E), dtype=torch.bfloat16, device=dev)
        nb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        _, keys_np = synth.host_ids_keys(synth.workload("layer27b"))
        keys = torch.from_numpy(keys_np).to(dev)
        proj = torch.empty(129280, dtype=torch.int32, device=dev)
        vb = eg.engram_workspace_size(None, eg.WS_VOCAB, 129280)
        eg.engram_build_vocab_proj(keys, 129280, proj, torch.empty(vb, dtype=torch.uint8, device=dev), vb)
        ids = torch.randint(0, 129280, (N,), generator=g, device=dev, dtype=torch.int32)
        state = torch.full((N, 2), cfg.V_c, dtype=torch.int32, device=dev)
        conv_state = torch.zeros((N, 1, 9 if a.dilated else 3, a.d), device=dev)
        idx = torch.empty((N, 1, a.heads), dtype=torch.int32, device=dev)

        def run():  # one decode step: hash and gather in one kernel, then the passes
            eg.engram_decode_step(cfg, proj, ids, state, idx, table, e, h, Wk, Wv, cw, conv_state,
                                  out, N, ws, nb)
    else:
        ids_np, keys_np = synth.host_ids_keys(synth.workload("layer27b"))
        keys = torch.from_numpy(keys_np).to(dev)
        proj = torch.empty(129280, dtype=torch.int32, device=dev)
        vb = eg.engram_workspace_size(None, eg.WS_VOCAB, 129280)
        vws = torch.empty(vb, dtype=torch.uint8, device=dev)
        eg.engram_build_vocab_proj(keys, 129280, proj, vws, vb)
        ids = torch.from_numpy(ids_np.reshape(-1)[:N].copy()).to(dev)
        idx = torch.empty((N, a.heads), dtype=torch.int32, device=dev)

        def run():
            eg.engram_hash_indices(cfg, proj, ids, B, T, None, idx)

    for r in range(a.reps):
        ev0.record()
        run()
        ev1.record()
        torch.cuda.synchronize()
        print(f"{a.kernel} rep {r}: {ev0.elapsed_time(ev1) * 1e3:.1f} us")
    if a.kernel == "hostcache":
        print(f"hostcache: {n_c} cached rows, {int(n_miss.item())} of {N * a.heads} "
              "(token, head) rows from host memory")
    st = eg.engram_get_status()
    if st != 0:
        raise SystemExit(f"device status word {st}")


def _tiny_step(dev):
    """The tiny fp32 layer (1 x 64 tokens, d 64, 4 heads x 16 dims): hash,
    forward with the gather, backward with the sparse table gradient."""
    w = synth.workload("tiny")
    inp = synth.host_inputs(w)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    keys = t(inp["keys"])
    proj = torch.empty(w.V, dtype=torch.int32, device=dev)
    vb = eg.engram_workspace_size(None, eg.WS_VOCAB, w.V)
    V_c = eg.engram_build_vocab_proj(keys, w.V, proj,
                                     torch.empty(vb, dtype=torch.uint8, device=dev), vb)
    cfg = eg.make_cfg(w.K, w.D_h, w.d, w.M, w.V, V_c, eg.F32, w.rows, inp["mult"])
    N, E = w.N, w.E
    ids, table = t(inp["ids"]), t(np.concatenate([x.reshape(-1) for x in inp["tables"]]))
    h, Wk, Wv, dout = t(inp["h"]), t(inp["Wk"]), t(inp["Wv"]), t(inp["dout"])
    cw = t(np.asarray(inp["conv_w"], np.float32).reshape(-1))
    idx = torch.empty((w.B, w.T, w.J), dtype=torch.int32, device=dev)
    e = torch.empty((N, E), device=dev)
    out = torch.empty((N, w.M, w.d), device=dev)
    saved = torch.empty(eg.engram_saved_size(cfg, N), dtype=torch.uint8, device=dev)
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    fws = torch.empty(fb, dtype=torch.uint8, device=dev)
    bb = eg.engram_workspace_size(cfg, eg.WS_BACKWARD, N)
    bws = torch.empty(bb, dtype=torch.uint8, device=dev)
    dh = torch.empty((N, w.M, w.d), device=dev)
    dWk, dWv = torch.empty((w.M, w.d, E), device=dev), torch.empty((w.d, E), device=dev)
    dcw = torch.empty(eg.engram_param_floats(cfg), device=dev)
    keys_out = torch.empty(N * w.J, dtype=torch.int64, device=dev)
    rows_out = torch.empty((N * w.J, w.D_h), device=dev)
    nu = torch.zeros(1, dtype=torch.int32, device=dev)

    def run():
        eg.engram_hash_indices(cfg, proj, ids, w.B, w.T, None, idx)
        eg.engram_forward(cfg, idx, table, e, h, Wk, Wv, cw, None, out, saved, w.B, w.T, fws, fb)
        eg.engram_backward(cfg, idx, e, h, Wk, Wv, cw, saved, dout, dh, dWk, dWv, dcw, None,
                           keys_out, rows_out, nu, w.B, w.T, bws, bb)
    return run


if __name__ == "__main__":
    main()
