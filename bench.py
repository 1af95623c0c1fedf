"""Throughput of the Engram layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the layer's hot path over one batch of the 27B-shaped
workload (8 sequences x 4,096 tokens, d 2,560, 16 hash heads x 80 dims over a
5.7B-parameter bf16 table): compress + n-gram + hash, row gather, then the two
fused tensor-core passes (gate partials; gate + value + causal conv +
residual).  Inputs are seeded and synthetic and stay resident in HBM; the
table (11.4 GB) and the hidden state (168 MB) exceed the 126 MB L2, so no
flush is needed between steps.

With N > 1 (torchrun), every rank runs an independent replica on its own
batch (weak scaling, no collective on the data path); timing is the max over
ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("Engram layer tokens/s (fwd, fwd+bwd) and achieved HBM GB/s / tensor-pipe % of "
          "B200 peak")
WORKLOAD = "layer27b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- distribution

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def dist_init(backend: str):
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank


def barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float) -> float:
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each replica draws its own token batch."""
    return base + 7919 * rank


def aggregate_rate(units_per_rank: int, world: int, steps: int, elapsed_ms_max: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time."""
    return units_per_rank * world * steps / (elapsed_ms_max / 1e3)


# ---------------------------------------------------------------- peaks, clocks

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gpu_uuid(local: int):
    """'GPU-…' identifier of the CUDA device, for nvidia-smi and NVML (whose
    indices need not follow CUDA_VISIBLE_DEVICES)."""
    try:
        import torch
        return "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:  # noqa: BLE001
        return None


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons during the timed region.

    Two sources: nvidia-smi every 100 ms (the standard record), and an NVML
    poller every ~2 ms restricted to the window between begin() and end(),
    which a timed region of tens of milliseconds needs to be sampled at all.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {4: "sw_power_cap", 8: "hw_slowdown", 32: "sw_thermal_slowdown",
               64: "hw_thermal_slowdown", 128: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.uuid = gpu_uuid(gpu_index)
        self.proc = None
        self.path = None
        self.nv = []
        self.window = None
        self._stop = False
        self._thread = None

    def _poll(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid
                 else pynvml.nvmlDeviceGetHandleByIndex(self.gpu))
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            while not self._stop:
                t = time.perf_counter()
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.nv.append((t, sm, rs, pw))
                time.sleep(0.002)
            pynvml.nvmlShutdown()
        except Exception:  # noqa: BLE001 -- the nvidia-smi record remains
            pass

    def begin(self):
        self.window = [time.perf_counter(), None]

    def end(self):
        if self.window is not None:
            self.window[1] = time.perf_counter()

    def __enter__(self):
        import threading
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid or self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def _smi_rows(self):
        rows = []
        if self.proc is None or self.path is None:
            return rows
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                     power=float(parts[3]), hw=parts[5], hwt=parts[6],
                                     swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        return rows

    def summary(self):
        rows = self._smi_rows()
        reasons = set()
        for r in rows:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["pcap"] == "Active":
                reasons.add("sw_power_cap")
        out = {}
        if rows:
            loaded = [r for r in rows if r["power"] > 250.0] or rows
            out = {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                   "sm_max_mhz": max(r["smax"] for r in rows),
                   "smi_samples": len(rows), "smi_samples_under_load": len(loaded)}
        win = [x for x in self.nv if self.window and self.window[1] is not None
               and self.window[0] <= x[0] <= self.window[1]]
        if win:
            for _, _, rs, _ in win:
                for bit, name in self.REASONS.items():
                    if rs & bit:
                        reasons.add(name)
            sms = [x[1] for x in win]
            out.update({"sm_mhz": statistics.median(sms), "sm_min_mhz": min(sms),
                        "sm_max_mhz": getattr(self, "smax", out.get("sm_max_mhz")),
                        "nvml_samples_in_timed_region": len(win),
                        "power_w_median": statistics.median(x[3] for x in win)})
        if not out:
            return None
        out["reasons"] = sorted(reasons)
        return out


# ---------------------------------------------------------------- CPU oracle

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class single_thread:
    """The oracle runs single-threaded: numpy's BLAS pool is held to one
    thread for the duration (threadpoolctl)."""

    def __enter__(self):
        try:
            from threadpoolctl import threadpool_limits
            self._lim = threadpool_limits(limits=1)
        except Exception:  # noqa: BLE001 -- numpy without a BLAS pool runs on one thread
            self._lim = None
        return self

    def __exit__(self, *a):
        if self._lim is not None:
            self._lim.unregister()


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return 1


def time_oracle(fn, min_s: float = 1.0):
    """Seconds per call of `fn` on one thread: one untimed call, then calls
    until min_s has passed."""
    with single_thread():
        fn()
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            el = time.perf_counter() - t0
            if el >= min_s:
                break
        return el / n, oracle_threads()


def oracle_sample(w, ids, keys, mult, head_rows_fn, dense_host, n_seq: int, n_tok: int):
    """The oracle end to end (hash, gather, fusion) on the first
    `n_tok` tokens of each of the first `n_seq` sequences of the batch, on
    one thread.

    `head_rows_fn(j, slots)` supplies rows `slots` of head j's table as
    [len(slots), D_h] float64; the oracle then gathers from a compact table
    of just the rows the sample touches.  Supplying the rows is data
    movement, not the method, and stays outside the timed spans.
    Returns (tokens, seconds, threads)."""
    from oracle import engram_oracle as O
    proj, V_c = O.build_vocab_proj(keys)     # one-time set-up, untimed on both sides
    with single_thread():
        threads = oracle_threads()
        t0 = time.perf_counter()
        sub = np.ascontiguousarray(ids[:n_seq, :n_tok])
        idx = O.hash_indices(proj, sub, mult, np.array(w.rows), w.K, V_c).reshape(-1, w.J)
        sec = time.perf_counter() - t0
        tables, local = [], np.empty_like(idx)
        for j in range(w.J):
            u, inv = np.unique(idx[:, j], return_inverse=True)
            tables.append(head_rows_fn(j, u))
            local[:, j] = inv.reshape(-1)
        h = dense_host["h"][: n_seq * n_tok]
        t1 = time.perf_counter()
        e = O.gather(local, tables)
        O.layer_forward(e, h, dense_host["Wk"], dense_host["Wv"], dense_host["conv_w"], n_tok)
        sec += time.perf_counter() - t1
    return n_seq * n_tok, sec, threads


def graph_kernel_nodes(g):
    """Kernel nodes of a captured graph (kept with keep_graph=True), or None."""
    try:
        from cuda.bindings import runtime as rt
        graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(graph, numNodes=0)
        err, nodes, n = rt.cudaGraphGetNodes(graph, numNodes=n)
        k = 0
        for nd in nodes:
            err, t = rt.cudaGraphNodeGetType(nd)
            if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                k += 1
        return k
    except Exception:  # noqa: BLE001 -- reported as unknown
        return None


# ---------------------------------------------------------------- our path

def run_ours(args):
    import torch

    from hashed_gram_conditional_engram_b200 import build as _b
    _b.build()
    from hashed_gram_conditional_engram_b200 import engram as eg
    from hashed_gram_conditional_engram_b200 import synth

    _, _, local = dist_env()
    torch.cuda.set_device(local)  # before the process group, so NCCL binds this GPU
    ws_, rank = dist_init("nccl")
    dev = torch.device("cuda", local)
    w = synth.workload(WORKLOAD)

    # ---- inputs (seeded, synthetic, resident in HBM)
    w_rank = synth.Workload(**{**w.__dict__, "seed": rank_seed(w.seed, rank)})
    ids_np = synth.host_ids_keys(w_rank)[0]
    keys_np = synth.host_ids_keys(w)[1]
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    table = synth.device_table(w, device=dev)
    dense = synth.device_dense(w, device=dev)
    keys = torch.from_numpy(keys_np).to(dev)
    proj = torch.empty(w.V, dtype=torch.int32, device=dev)
    vb = eg.engram_workspace_size(None, eg.WS_VOCAB, w.V)
    vws = torch.empty(vb, dtype=torch.uint8, device=dev)
    V_c = eg.engram_build_vocab_proj(keys, w.V, proj, vws, vb)
    del vws
    cfg = eg.make_cfg(w.K, w.D_h, w.d, 1, w.V, V_c, eg.BF16, w.rows, mult)
    N = w.N
    ids = torch.from_numpy(ids_np).to(dev)
    idx = torch.empty((w.B, w.T, w.J), dtype=torch.int32, device=dev)
    e = torch.empty((N, w.E), dtype=torch.bfloat16, device=dev)
    out = torch.empty((w.B, w.T, 1, w.d), dtype=torch.bfloat16, device=dev)
    saved = torch.empty(eg.engram_saved_size(cfg, N), dtype=torch.uint8, device=dev)
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    fws = torch.empty(fb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        eg.engram_hash_indices(cfg, proj, ids, w.B, w.T, None, idx, stream)
        if ev is not None:
            ev[1].record(stream)
        eg.engram_gather(cfg, idx, table, N, e, stream)
        if ev is not None:
            ev[2].record(stream)
        eg.engram_forward(cfg, idx, None, e, dense["h"], dense["Wk"], dense["Wv"],
                          dense["conv_w"], None, out, saved, w.B, w.T, fws, fb, stream)
        if ev is not None:
            ev[3].record(stream)

    for i in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if eg.engram_get_status(stream) != 0:
        raise RuntimeError("device status word set during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        clk.begin()
        start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        end.record(stream)
        torch.cuda.synchronize()
        clk.end()
        barrier()
    clocks = clk.summary() or {}
    elapsed_ms = start.elapsed_time(end)
    t_hash = sum(ev[0].elapsed_time(ev[1]) for ev in evs) / args.steps
    t_gather = sum(ev[1].elapsed_time(ev[2]) for ev in evs) / args.steps
    t_fuse = sum(ev[2].elapsed_time(ev[3]) for ev in evs) / args.steps
    if eg.engram_get_status(stream) != 0:
        raise RuntimeError("device status word set during timing")
    elapsed_ms = max_over_ranks(elapsed_ms)
    ms_per_step = elapsed_ms / args.steps
    value = aggregate_rate(N, ws_, args.steps, elapsed_ms)

    # ---- the gather alone: back to back (the slots and whatever rows the
    # previous call left in L2 stay warm) and with a 256 MB memset between
    # calls (L2 flushed)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    gev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    t_warm, t_cold = [], []
    for k in range(21):
        flushed = k % 2 == 1
        if flushed:
            flush.zero_()
        gev[0].record(stream)
        eg.engram_gather(cfg, idx, table, N, e, stream)
        gev[1].record(stream)
        torch.cuda.synchronize()
        (t_cold if flushed else t_warm).append(gev[0].elapsed_time(gev[1]))
    del flush
    gather_l2 = {"warm_us": float(np.median(t_warm[1:])) * 1e3,
                 "l2_flushed_us": float(np.median(t_cold)) * 1e3,
                 "what": "engram_gather alone, median of 10 calls each: back to back, and "
                         "after a 256 MB memset (L2 flushed)"}

    # ---- end to end through the public API with host buffers.  Each step
    # uploads its ids and h from pinned host memory, runs hash + forward and
    # reads its output back.  Steps are double-buffered over three streams
    # (upload, compute, download), as a serving loop would run them: PCIe is
    # full duplex, so step k+1's upload, step k's compute and step k-1's
    # download overlap.
    ids_h = torch.from_numpy(ids_np).pin_memory()
    h_h = dense["h"].cpu().pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    ids_d = [torch.empty_like(ids) for _ in range(2)]
    h_d = [torch.empty_like(dense["h"]) for _ in range(2)]
    out_d = [torch.empty_like(out) for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    for k in range(2):  # every event recorded once, so the first waits pass
        for ev in (ev_comp[k], ev_down[k]):
            ev.record(stream)

    def e2e_step(k):
        b = k % 2
        up.wait_event(ev_comp[b])         # step k-2's compute has read h_d[b]
        with torch.cuda.stream(up):
            ids_d[b].copy_(ids_h, non_blocking=True)
            h_d[b].copy_(h_h, non_blocking=True)
        ev_up[b].record(up)
        stream.wait_event(ev_up[b])
        stream.wait_event(ev_down[b])     # step k-2's output has left out_d[b]
        eg.engram_hash_indices(cfg, proj, ids_d[b], w.B, w.T, None, idx, stream)
        eg.engram_forward(cfg, idx, table, e, h_d[b], dense["Wk"], dense["Wv"], dense["conv_w"],
                          None, out_d[b], saved, w.B, w.T, fws, fb, stream)
        ev_comp[b].record(stream)
        down.wait_event(ev_comp[b])
        with torch.cuda.stream(down):
            out_h[b].copy_(out_d[b], non_blocking=True)
        ev_down[b].record(down)

    for k in range(2):
        e2e_step(k)
    e2e_steps = max(4, min(args.steps, 20))
    barrier()
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(up)
    for k in range(e2e_steps):
        e2e_step(k)
    e2.record(down)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(s2.elapsed_time(e2))
    e2e_value = aggregate_rate(N, ws_, e2e_steps, e2e_ms)
    h2d = ids_h.numel() * 4 + h_h.numel() * 2
    d2h = out_h[0].numel() * 2
    if not torch.equal(out_d[(e2e_steps - 1) % 2], out):
        raise RuntimeError("end-to-end output differs from the device-resident step")

    # ---- roofline of the dominant kernel (the two fused tensor-core passes)
    peaks, peak_src = load_peaks()
    flops = 2 * 2.0 * N * w.E * w.d            # k and v projections, algorithmic
    achieved = flops / (t_fuse / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    traffic = None
    tp = os.path.join(ROOT, "profiles", "traffic_layer27b.json")
    if os.path.exists(tp):
        # the counters apply only to the kernel source they were taken from
        import hashlib
        with open(tp) as f:
            rec = json.load(f)
        h_ = hashlib.sha1()
        for rel in rec.get("source_files", []):
            with open(os.path.join(ROOT, rel), "rb") as f:
                h_.update(f.read())
        if rec.get("source_files") and rec.get("source_sha1") == h_.hexdigest():
            traffic = rec.get("fused_tc_traffic_bytes_per_step")

    line = None
    if rank == 0:
        cpu = None
        if ws_ == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline_ours(w, ids_np, keys_np, mult, table, dense)
        extras = {}
        if ws_ == 1 and not args.no_extras:
            for name, fn in (("decode", bench_decode), ("hosttable", bench_hosttable),
                             ("fwd_bwd", bench_train_step), ("tiny", bench_tiny),
                             ("tiny_all_variants",
                              lambda d_: bench_tiny(d_, flags=30)),  # dilated, prenorm, per-branch, scales
                             ("fwd_bwd_27b", bench_fwd_bwd_27b)):
                try:
                    extras[name] = fn(dev)
                except Exception as ex:  # noqa: BLE001 -- reported, not hidden
                    extras[name] = {"error": f"{type(ex).__name__}: {ex}"}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Zipf(1.1) ids, N(0,0.02) bf16 table and weights, N(0,1) h)",
            "config": {
                "workload": "layer27b: 27B-shaped Engram layer forward, 8 x 4,096 tokens, "
                            "d_model 2,560, orders {2,3} x 8 heads x 80 dims, 16 primes "
                            "<= 4,450,001 (5.7B bf16 params), vocab 129,280 -> 99,546",
                "global_batch": N * ws_, "seq_len": w.T, "parallelism": f"dp{ws_} (replicas)",
                "l2": "inputs larger than L2 (table 11.4 GB, h 168 MB per step); no flush",
            },
            "breakdown_ms": {"hash": t_hash, "gather": t_gather, "fused_tc_passes": t_fuse},
            "gather_gbs": (N * w.J * 4 + N * w.J * w.D_h * 2 + N * w.E * 2) / (t_gather / 1e3) / 1e9,
            "gather_alone": gather_l2,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "kernel": "engram_forward(table=NULL): tc_fused_kernel pass K, gate kernel, tc_fused_kernel pass V",
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         # the step loop runs the tensor pipe for tens of ms under the
                         # 1 kW cap: the sustained figure is the one it can hold
                         "peak_sustained": peak_sus, "frac_of_sustained": achieved / peak_sus},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": 5 * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "other_workloads": extras,
        }
    barrier()
    return line


def cpu_baseline_ours(w, ids_np, keys_np, mult, table, dense):
    """The oracle on a bounded sample of the same workload: the first
    sequence of the batch (4,096 tokens), end to end, on one thread."""
    import torch
    base = np.concatenate([[0], np.cumsum(w.rows)[:-1]])
    n_seq = 1
    dense_host = {
        "h": dense["h"][:n_seq].reshape(-1, 1, w.d).double().cpu().numpy(),
        "Wk": dense["Wk"].double().cpu().numpy(),
        "Wv": dense["Wv"].double().cpu().numpy(),
        "conv_w": dense["conv_w"].double().cpu().numpy(),
    }

    def rows_fn(j, slots):
        r = torch.from_numpy(base[j] + slots.astype(np.int64)).to(table.device)
        return table.view(-1, w.D_h).index_select(0, r).double().cpu().numpy()

    tok, sec, thr = oracle_sample(w, ids_np, keys_np, mult, rows_fn, dense_host, n_seq, w.T)
    return {"value": tok / sec, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"first sequence of the batch ({tok} tokens), oracle end to end in fp64 "
                      f"on one thread ({sec:.1f} s)"}


# ---------------------------------------------------------------- other workloads

def _time_loop(fn, steps, warmup, stream):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def _graph_time(fn, steps, warmup, stream, nodes=None):
    """The same step captured once into a CUDA graph and replayed; with a
    list `nodes`, the graph's kernel-node count is appended to it."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g, stream=stream):
        fn()
    if nodes is not None:
        nodes.append(graph_kernel_nodes(g))
    g.instantiate()
    return _time_loop(g.replay, steps, warmup, stream)


_FLOOR = {}


def launch_floor_us(dev, stream):
    """Device time per kernel node of a graph of 200 one-element kernels:
    the floor a chain of dependent launches cannot go below."""
    import torch
    if "us" not in _FLOOR:
        x = torch.zeros(1, device=dev)

        def chain():
            for _ in range(200):
                x.add_(1.0)

        with torch.cuda.stream(stream):
            _FLOOR["us"] = _graph_time(chain, 20, 2, stream) * 1e3 / 200
    return _FLOOR["us"]


def latency_roofline(dev, stream, us_per_call, kernels):
    """Launch-latency roofline of a small step: its kernel count times the
    per-kernel floor of a graph, against the measured time."""
    floor = launch_floor_us(dev, stream)
    if not kernels:
        return {"bound": "latency", "achieved": us_per_call, "peak": None, "unit": "us",
                "frac": None, "kernels_per_step": kernels, "floor_us_per_kernel": floor}
    peak = kernels * floor
    return {"bound": "latency", "achieved": us_per_call, "peak": peak, "unit": "us",
            "frac": peak / us_per_call, "traffic": None, "kernels_per_step": kernels,
            "floor_us_per_kernel": floor,
            "how": "peak = kernels in the step's CUDA graph x device time per node of a graph of "
                   "200 one-element kernels; frac = peak / measured (1.0 = launch-bound floor)"}


def bench_fwd_bwd_27b(dev, steps=10):
    """Training step of the 27B-shaped layer (8 x 4,096 tokens, d 2,560, 16 x
    80 dims, 5.7B-parameter bf16 table): hash, forward (gather, fused passes,
    alpha, k and v saved), backward (bf16: elementwise kernels, tensor-core
    GEMMs, sparse table gradient); the same with k and v recomputed in the
    backward instead of saved; with the dilated conv (taps 3, 6 and 9
    tokens back); and with the pre-conv RMSNorm."""
    keys = ("ms_per_step", "fwd_bwd_tokens_per_s", "breakdown_ms", "roofline")
    kept = _fwd_bwd_27b_run(dev, steps, save_kv=True, cpu=True)
    recomputed = _fwd_bwd_27b_run(dev, steps, save_kv=False)
    kept["recompute_kv"] = {k: recomputed[k] for k in keys}
    from hashed_gram_conditional_engram_b200 import engram as eg
    dilated = _fwd_bwd_27b_run(dev, steps, save_kv=True, variant=eg.CONV_DILATED)
    kept["dilated_conv"] = {k: dilated[k] for k in keys}
    prenorm = _fwd_bwd_27b_run(dev, steps, save_kv=True, variant=eg.CONV_PRENORM)
    kept["prenorm_conv"] = {k: prenorm[k] for k in keys}
    return kept


def cpu_baseline_fwd_bwd_27b(w, ids_np, keys_np, mult, table, dense, dout, n_tok=512):
    """The oracle's training step on the first n_tok tokens of the first
    sequence: hash, gather, forward, backward and the table gradient, fp64,
    one thread (the rows the sample touches are fetched outside the timing)."""
    import torch
    from oracle import engram_oracle as O
    proj, V_c = O.build_vocab_proj(keys_np)
    base = np.concatenate([[0], np.cumsum(w.rows)[:-1]])
    ids = np.ascontiguousarray(ids_np[:1, :n_tok])
    idx = O.hash_indices(proj, ids, mult, np.array(w.rows), w.K, V_c).reshape(-1, w.J)
    tables, local = [], np.empty_like(idx)
    for j in range(w.J):
        u, inv = np.unique(idx[:, j], return_inverse=True)
        r = torch.from_numpy(base[j] + u.astype(np.int64)).to(table.device)
        tables.append(table.view(-1, w.D_h).index_select(0, r).double().cpu().numpy())
        local[:, j] = inv.reshape(-1)
    h = dense["h"][:1, :n_tok].reshape(n_tok, 1, w.d).double().cpu().numpy()
    Wk, Wv = dense["Wk"].double().cpu().numpy(), dense["Wv"].double().cpu().numpy()
    cw = dense["conv_w"].double().cpu().numpy()
    u = dout[:n_tok].double().cpu().numpy()

    def run():
        O.hash_indices(proj, ids, mult, np.array(w.rows), w.K, V_c)
        e = O.gather(local, tables)
        g = O.layer_backward(e, h, Wk, Wv, cw, n_tok, u)
        O.table_grad_segments_fast(local, g["de"].astype(np.float32),
                                   [t.shape[0] for t in tables], w.D_h)

    sec, thr = time_oracle(run, min_s=3.0)
    return {"value": n_tok / sec, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"first {n_tok} tokens of sequence 0: hash, gather, forward, backward, "
                      f"table gradient in fp64 on one thread ({sec:.2f} s per call)"}


def _fwd_bwd_27b_run(dev, steps, save_kv, variant=0, cpu=False):
    import torch
    from hashed_gram_conditional_engram_b200 import engram as eg
    from hashed_gram_conditional_engram_b200 import synth
    w = synth.workload(WORKLOAD)
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    ids_np, keys_np = synth.host_ids_keys(w)
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    table = synth.device_table(w, device=dev)
    dense = synth.device_dense(w, device=dev)
    keys = torch.from_numpy(keys_np).to(dev)
    proj = torch.empty(w.V, dtype=torch.int32, device=dev)
    vb = eg.engram_workspace_size(None, eg.WS_VOCAB, w.V)
    V_c = eg.engram_build_vocab_proj(keys, w.V, proj, torch.empty(vb, dtype=torch.uint8, device=dev), vb)
    cfg = eg.make_cfg(w.K, w.D_h, w.d, 1, w.V, V_c, eg.BF16, w.rows, mult,
                      flags=(eg.SAVE_KV if save_kv else 0) | variant)
    N, E = w.N, w.E
    ids = torch.from_numpy(ids_np).to(dev)
    idx = torch.empty((w.B, w.T, w.J), dtype=torch.int32, device=dev)
    e = torch.empty((N, E), dtype=torch.bfloat16, device=dev)
    out = torch.empty((N, 1, w.d), dtype=torch.bfloat16, device=dev)
    saved = torch.empty(eg.engram_saved_size(cfg, N), dtype=torch.uint8, device=dev)
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
    fws = torch.empty(fb, dtype=torch.uint8, device=dev)
    bb = eg.engram_workspace_size(cfg, eg.WS_BACKWARD, N)
    bws = torch.empty(bb, dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(27)
    dout = torch.randn((N, 1, w.d), generator=g, device=dev)
    dh = torch.empty((N, 1, w.d), device=dev)
    dWk, dWv = torch.empty((1, w.d, E), device=dev), torch.empty((w.d, E), device=dev)
    dcw = torch.empty((w.d, 4), device=dev)
    keys_out = torch.empty(N * w.J, dtype=torch.int64, device=dev)
    rows_out = torch.empty((N * w.J, w.D_h), device=dev)
    nu = torch.zeros(1, dtype=torch.int32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def step(mark=False):
        if mark:
            ev[0].record(s)
        eg.engram_hash_indices(cfg, proj, ids, w.B, w.T, None, idx, s)
        eg.engram_forward(cfg, idx, table, e, dense["h"], dense["Wk"], dense["Wv"],
                          dense["conv_w"], None, out, saved, w.B, w.T, fws, fb, s)
        if mark:
            ev[1].record(s)
        eg.engram_backward(cfg, idx, e, dense["h"], dense["Wk"], dense["Wv"], dense["conv_w"],
                           saved, dout, dh, dWk, dWv, dcw, None, keys_out, rows_out, nu,
                           w.B, w.T, bws, bb, s)
        if mark:
            ev[2].record(s)

    with torch.cuda.stream(s):
        ms = _time_loop(step, steps, 3, s)
        step(mark=True)
        torch.cuda.synchronize()
    if eg.engram_get_status(s) != 0:
        raise RuntimeError("device status word set in the 27B-shaped training step")
    # dense contractions of one step: forward k and v; backward [dW_k; dW_v]
    # and de (K = 2d), and [k | v] again unless the forward kept them
    flops = 2.0 * N * E * w.d * 2 + 2.0 * N * E * (2 * w.d) * (2 if save_kv else 3)
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = flops / (ms / 1e3) / 1e12
    cpu_line = None
    if cpu:
        cpu_line = cpu_baseline_fwd_bwd_27b(w, ids_np, keys_np, mult, table, dense, dout)
    t_bwd = ev[1].elapsed_time(ev[2])
    del table, dense, bws, fws
    torch.cuda.empty_cache()
    out_line = {
        "workload": "layer27b training step: 8 x 4,096 tokens, d 2,560, 16 heads x 80 dims, "
                    "5.7B bf16 params; forward (hash, gather, fused passes"
                    + (", k and v saved" if save_kv else "") + ") + bf16 backward",
        "fwd_bwd_tokens_per_s": N / (ms / 1e3), "ms_per_step": ms,
        "breakdown_ms": {"forward": ev[0].elapsed_time(ev[1]), "backward": t_bwd},
        # the step's dense flops over the whole step's time (the elementwise
        # kernels between the GEMMs included): a floor on the GEMMs' own rate,
        # whose kernel times are in the committed launch list
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "what": "all dense GEMM flops of the step / whole step time",
                     "flops_per_step": flops,
                     "peak_source": f"{peak_src} bf16_tflops_sustained"},
    }
    if cpu_line is not None:
        out_line["cpu_baseline"] = cpu_line
    return out_line


def bench_tiny(dev, flags=0):
    """One fp32 layer (1 x 64 tokens, d 64, 4 heads x 16 dims): hash, forward
    with the gather, backward with the sparse table gradient, per call; with
    `flags`, the formulation variants (their extra parameters: conv weights
    repeated per branch, norm scales 1 + N(0, 0.1))."""
    import torch
    from hashed_gram_conditional_engram_b200 import engram as eg
    from hashed_gram_conditional_engram_b200 import synth
    w = synth.workload("tiny")
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    inp = synth.host_inputs(w)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    keys = t(inp["keys"])
    proj = torch.empty(w.V, dtype=torch.int32, device=dev)
    vb = eg.engram_workspace_size(None, eg.WS_VOCAB, w.V)
    V_c = eg.engram_build_vocab_proj(keys, w.V, proj, torch.empty(vb, dtype=torch.uint8, device=dev), vb)
    cfg = eg.make_cfg(w.K, w.D_h, w.d, w.M, w.V, V_c, eg.F32, w.rows, inp["mult"], flags=flags)
    N, E = w.N, w.E
    ids, table = t(inp["ids"]), t(np.concatenate([x.reshape(-1) for x in inp["tables"]]))
    block = np.asarray(inp["conv_w"], np.float32).reshape(-1)
    if flags & eg.CONV_PER_BRANCH:
        block = np.tile(block, w.M)
    n_par = eg.engram_param_floats(cfg)
    if n_par > block.size:
        rng = np.random.default_rng(w.seed + 9)
        block = np.r_[block, 1.0 + 0.1 * rng.standard_normal(n_par - block.size)].astype(np.float32)
    h, Wk, Wv, cw, dout = t(inp["h"]), t(inp["Wk"]), t(inp["Wv"]), t(block), t(inp["dout"])
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
    dcw = torch.empty(n_par, device=dev)
    keys_out = torch.empty(N * w.J, dtype=torch.int64, device=dev)
    rows_out = torch.empty((N * w.J, w.D_h), device=dev)
    nu = torch.zeros(1, dtype=torch.int32, device=dev)

    def fwd():
        eg.engram_hash_indices(cfg, proj, ids, w.B, w.T, None, idx, s)
        eg.engram_forward(cfg, idx, table, e, h, Wk, Wv, cw, None, out, saved, w.B, w.T, fws, fb, s)

    def step():
        fwd()
        eg.engram_backward(cfg, idx, e, h, Wk, Wv, cw, saved, dout, dh, dWk, dWv, dcw, None,
                           keys_out, rows_out, nu, w.B, w.T, bws, bb, s)

    nodes = []
    with torch.cuda.stream(s):
        f_eager = _time_loop(fwd, 200, 5, s)
        fb_eager = _time_loop(step, 200, 5, s)
        fb_graph = _graph_time(step, 500, 5, s, nodes)
    if eg.engram_get_status(s) != 0:
        raise RuntimeError("device status word set in the tiny layer")
    from oracle import engram_oracle as O
    proj_ref, V_c_ref = O.build_vocab_proj(inp["keys"])
    tables64 = [np.asarray(x, np.float64) for x in inp["tables"]]

    def oracle_step():
        idx_r = O.hash_indices(proj_ref, inp["ids"], inp["mult"], inp["rows"], w.K, V_c_ref)
        e_r = O.gather(idx_r.reshape(-1, w.J), tables64)
        h_r = inp["h"].reshape(N, w.M, w.d)
        if flags:
            g_r = O.layer_backward_v(e_r, h_r, inp["Wk"], inp["Wv"], block, w.T,
                                     inp["dout"].reshape(N, w.M, w.d), flags)
        else:
            g_r = O.layer_backward(e_r, h_r, inp["Wk"], inp["Wv"], inp["conv_w"], w.T,
                                   inp["dout"].reshape(N, w.M, w.d))
        O.table_grad_segments_fast(idx_r.reshape(-1, w.J), g_r["de"].astype(np.float32),
                                   w.rows, w.D_h)

    sec, thr = time_oracle(oracle_step)
    return {"workload": "tiny: 1 x 64 tokens, d 64, K 2 x 1,009 x 16, fp32 (fp64 arithmetic), "
                        "one layer" + (f", variant flags {flags}" if flags else ""),
            "us_per_fwd_call_eager": f_eager * 1e3, "us_per_fwd_bwd_call_eager": fb_eager * 1e3,
            "us_per_fwd_bwd_graph": fb_graph * 1e3,
            "fwd_bwd_tokens_per_s": w.N / (fb_graph / 1e3),
            "roofline": latency_roofline(dev, s, fb_graph * 1e3, nodes[0] if nodes else None),
            "cpu_baseline": {"value": w.N / sec, "unit": "tokens/s", "cores": thr,
                             "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": "the whole workload (64 tokens): hash, gather, forward, "
                                       f"backward, table gradient in fp64 ({sec * 1e3:.1f} ms "
                                       "per call, one thread)"}}


def bench_train_step(dev):
    """Training step of the two-layer, 4-branch workload (fp32, 64 tokens):
    forward of the layers at 2 and 6, backward of both with the sparse table
    gradients."""
    import torch
    from hashed_gram_conditional_engram_b200 import engram as eg
    from hashed_gram_conditional_engram_b200 import synth
    w = synth.workload("train")
    s = torch.cuda.Stream(dev)          # graph capture needs a non-default stream
    s.wait_stream(torch.cuda.current_stream(dev))
    layers = []
    for li in (2, 6):
        inp = synth.host_inputs(w, layer=li)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
        keys = t(inp["keys"])
        proj = torch.empty(w.V, dtype=torch.int32, device=dev)
        vb = eg.engram_workspace_size(None, eg.WS_VOCAB, w.V)
        V_c = eg.engram_build_vocab_proj(keys, w.V, proj, torch.empty(vb, dtype=torch.uint8, device=dev), vb)
        cfg = eg.make_cfg(w.K, w.D_h, w.d, w.M, w.V, V_c, eg.F32, w.rows, inp["mult"])
        N, E = w.N, w.E
        L = dict(cfg=cfg, proj=proj, ids=t(inp["ids"]),
                 table=t(np.concatenate([x.reshape(-1) for x in inp["tables"]])),
                 Wk=t(inp["Wk"]), Wv=t(inp["Wv"]), cw=t(inp["conv_w"]),
                 idx=torch.empty((w.B, w.T, w.J), dtype=torch.int32, device=dev),
                 e=torch.empty((N, E), device=dev), out=torch.empty((N, w.M, w.d), device=dev),
                 saved=torch.empty(eg.engram_saved_size(cfg, N), dtype=torch.uint8, device=dev),
                 dh=torch.empty((N, w.M, w.d), device=dev), dWk=torch.empty((w.M, w.d, E), device=dev),
                 dWv=torch.empty((w.d, E), device=dev), dcw=torch.empty((w.d, 4), device=dev),
                 keys_out=torch.empty(N * w.J, dtype=torch.int64, device=dev),
                 rows_out=torch.empty((N * w.J, w.D_h), device=dev),
                 nu=torch.zeros(1, dtype=torch.int32, device=dev))
        L["fb"] = eg.engram_workspace_size(cfg, eg.WS_FORWARD, N)
        L["fws"] = torch.empty(L["fb"], dtype=torch.uint8, device=dev)
        L["bb"] = eg.engram_workspace_size(cfg, eg.WS_BACKWARD, N)
        L["bws"] = torch.empty(L["bb"], dtype=torch.uint8, device=dev)
        layers.append(L)
    h0 = torch.from_numpy(synth.host_inputs(w, layer=2)["h"]).to(dev)
    dout = torch.from_numpy(synth.host_inputs(w, layer=2)["dout"]).to(dev)

    def step():
        hin = h0
        for L in layers:
            eg.engram_hash_indices(L["cfg"], L["proj"], L["ids"], w.B, w.T, None, L["idx"], s)
            eg.engram_forward(L["cfg"], L["idx"], L["table"], L["e"], hin, L["Wk"], L["Wv"], L["cw"],
                              None, L["out"], L["saved"], w.B, w.T, L["fws"], L["fb"], s)
            L["hin"] = hin
            hin = L["out"]
        g = dout
        for L in reversed(layers):
            eg.engram_backward(L["cfg"], L["idx"], L["e"], L["hin"], L["Wk"], L["Wv"], L["cw"],
                               L["saved"], g, L["dh"], L["dWk"], L["dWv"], L["dcw"], None,
                               L["keys_out"], L["rows_out"], L["nu"], w.B, w.T, L["bws"], L["bb"], s)
            g = L["dh"]

    nodes = []
    with torch.cuda.stream(s):
        eager = _time_loop(step, 50, 5, s)
        graph = _graph_time(step, 200, 5, s, nodes)
    if eg.engram_get_status(s) != 0:
        raise RuntimeError("device status word set in the training step")
    from oracle import engram_oracle as O
    ref_layers = []
    for li in (2, 6):
        inp = synth.host_inputs(w, layer=li)
        proj_ref, V_c_ref = O.build_vocab_proj(inp["keys"])
        ref_layers.append((inp, proj_ref, V_c_ref, [np.asarray(x, np.float64) for x in inp["tables"]]))
    h0_r = synth.host_inputs(w, layer=2)["h"].reshape(w.N, w.M, w.d).astype(np.float64)
    dout_r = synth.host_inputs(w, layer=2)["dout"].reshape(w.N, w.M, w.d).astype(np.float64)

    def oracle_step():
        hin, saved_r = h0_r, []
        for inp, proj_ref, V_c_ref, tabs in ref_layers:
            idx_r = O.hash_indices(proj_ref, inp["ids"], inp["mult"], inp["rows"], w.K,
                                   V_c_ref).reshape(-1, w.J)
            e_r = O.gather(idx_r, tabs)
            f = O.layer_forward(e_r, hin, inp["Wk"], inp["Wv"], inp["conv_w"], w.T)
            saved_r.append((inp, idx_r, e_r, hin, f))
            hin = f["out"]
        g = dout_r
        for inp, idx_r, e_r, hin, f in reversed(saved_r):
            gr = O.layer_backward(e_r, hin, inp["Wk"], inp["Wv"], inp["conv_w"], w.T, g, fwd=f)
            O.table_grad_segments_fast(idx_r, gr["de"].astype(np.float32), w.rows, w.D_h)
            g = gr["dh"]

    sec, thr = time_oracle(oracle_step)
    return {"workload": "train: 1 x 64 tokens, d 64, 4 branches, Engram at layers 2 and 6, "
                        "K 2 x 1,009 x 16 per layer, fp32 (fp64 arithmetic)",
            "fwd_bwd_tokens_per_s": w.N / (graph / 1e3), "ms_per_step_graph": graph,
            "ms_per_step_eager": eager, "fwd_bwd_tokens_per_s_eager": w.N / (eager / 1e3),
            "roofline": latency_roofline(dev, s, graph * 1e3, nodes[0] if nodes else None),
            "cpu_baseline": {"value": w.N / sec, "unit": "tokens/s", "cores": thr,
                             "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": "the whole workload (64 tokens, both layers): forward "
                                       "and backward with the table gradients in fp64 "
                                       f"({sec * 1e3:.1f} ms per step, one thread)"}}


def bench_decode(dev):
    """Decode: 256 sequences x 1 token per step over the workload's 2,000
    steps of Zipf(1.1) ids, each step with its own pregenerated hidden state
    N(0, 1); d 4,096, K 8 x ~6.35M rows x 128 (13B bf16 parameters, 26 GB on
    the device), rolling n-gram and conv state.  One step = hash with the
    n-gram state and gather (one kernel), then pass K, the gate and pass V
    in one persistent launch (engram_decode_step).  All 2,000 steps are
    captured into one CUDA graph (each step reading its own ids and h rows),
    replayed once untimed and once timed from the same initial state."""
    import torch
    from hashed_gram_conditional_engram_b200 import engram as eg
    from hashed_gram_conditional_engram_b200 import synth
    w = synth.workload("decode")
    S = w.steps
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    ids_np, keys_np = synth.host_ids_keys(w)          # [2000, 256]
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    table = synth.device_table(w, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(41)
    Wk = (torch.randn((1, w.d, w.E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    Wv = (torch.randn((w.d, w.E), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    cw = torch.randn((w.d, 4), generator=g, device=dev) * 0.5
    hs = torch.empty((S, w.B, 1, 1, w.d), dtype=torch.bfloat16, device=dev)
    for a in range(0, S, 250):
        hs[a:a + 250] = torch.randn((min(250, S - a), w.B, 1, 1, w.d), generator=g,
                                    device=dev).to(torch.bfloat16)
    keys = torch.from_numpy(keys_np).to(dev)
    proj = torch.empty(w.V, dtype=torch.int32, device=dev)
    vb = eg.engram_workspace_size(None, eg.WS_VOCAB, w.V)
    V_c = eg.engram_build_vocab_proj(keys, w.V, proj, torch.empty(vb, dtype=torch.uint8, device=dev), vb)
    cfg = eg.make_cfg(w.K, w.D_h, w.d, 1, w.V, V_c, eg.BF16, w.rows, mult)
    ids = torch.from_numpy(ids_np).to(dev)
    state = torch.full((w.B, 2), V_c, dtype=torch.int32, device=dev)
    conv_state = torch.zeros((w.B, 1, 3, w.d), device=dev)
    e = torch.empty((w.B, w.E), dtype=torch.bfloat16, device=dev)
    out = torch.empty((w.B, 1, 1, w.d), dtype=torch.bfloat16, device=dev)
    fb = eg.engram_workspace_size(cfg, eg.WS_FORWARD, w.B)
    fws = torch.empty(fb, dtype=torch.uint8, device=dev)

    def step(k):  # hash + gather in one kernel, then the one-launch decode kernel
        eg.engram_decode_step(cfg, proj, ids[k], state, None, table, e, hs[k], Wk, Wv, cw,
                              conv_state, out, w.B, fws, fb, s)

    def reset():
        state.fill_(V_c)
        conv_state.zero_()

    def all_steps():
        for k in range(S):
            step(k)

    with torch.cuda.stream(s):
        for k in range(8):                       # set-up of the kernels on this device
            step(k)
        reset()
        torch.cuda.synchronize()
        # eager: one Python call pair per step (host-bound)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        all_steps()
        b.record(s)
        torch.cuda.synchronize()
        ms_eager = a.elapsed_time(b) / S
        reset()
        graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(graph, stream=s):
            all_steps()
        kernels = graph_kernel_nodes(graph)
        graph.instantiate()
        graph.replay()                           # untimed
        torch.cuda.synchronize()
        reset()
        torch.cuda.synchronize()
        a.record(s)
        graph.replay()
        b.record(s)
        torch.cuda.synchronize()
        ms_graph = a.elapsed_time(b) / S
    if eg.engram_get_status(s) != 0:
        raise RuntimeError("device status word set in decode")
    # algorithmic bytes per step: both weight matrices, the rows and indices,
    # ids and n-gram state, h and out, and the conv state read and rewritten
    # (three steps of history per feature, kept oldest first)
    wbytes = 2 * w.d * w.E * 2
    rbytes = w.B * w.J * (w.D_h * 2 + 4)
    sbytes = w.B * (4 + 2 * 4 * 2)
    hbytes = 2 * w.B * w.d * 2
    cbytes = 2 * w.B * 3 * w.d * 4
    step_bytes = wbytes + rbytes + sbytes + hbytes + cbytes
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = step_bytes / (ms_graph / 1e3) / 1e9
    cpu = cpu_baseline_decode(w, ids_np, keys_np, mult, table, Wk, Wv, cw, hs, V_c)
    del table, hs, graph
    torch.cuda.empty_cache()
    return {"workload": "decode: 256 sequences x 1 token per step, 2,000 steps of Zipf(1.1) ids "
                        "with fresh h per step, d_model 4,096, K 8 x 6.35M rows x 128 (13.0B bf16 "
                        "params), rolling n-gram and conv state",
            "tokens_per_s": w.B / (ms_graph / 1e3), "us_per_step_graph": ms_graph * 1e3,
            "us_per_step_eager": ms_eager * 1e3, "tokens_per_s_eager": w.B / (ms_eager / 1e3),
            "steps_timed": S, "kernels_per_step": (kernels / S) if kernels else None,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None,
                         "bytes_per_step": step_bytes,
                         "bytes_split": {"W_k + W_v": wbytes, "rows + idx": rbytes,
                                         "ids + ngram state": sbytes, "h + out": hbytes,
                                         "conv state read + write": cbytes},
                         "peak_source": f"{peak_src} hbm_gbs"},
            "cpu_baseline": cpu}


def cpu_baseline_decode(w, ids_np, keys_np, mult, table, Wk, Wv, cw, hs, V_c, n_steps=4):
    """The oracle's decode steps 0 .. n_steps-1 for all 256 sequences (hash
    with the rolling state, gather, gate, conv with the conv state), fp64 on
    one thread; the touched rows and the step's h are fetched outside the
    timing."""
    import torch
    from oracle import engram_oracle as O
    proj, V_c_ref = O.build_vocab_proj(keys_np)
    base = np.concatenate([[0], np.cumsum(w.rows)[:-1]])
    Wk_h, Wv_h = Wk.double().cpu().numpy(), Wv.double().cpu().numpy()
    cw_h = cw.double().cpu().numpy()
    # the rows the sample's steps touch, by a dry run of the hash
    st = np.full((w.B, 2), V_c_ref, np.int32)
    rows_of = []
    for k in range(n_steps):
        idx_k, st = O.hash_indices_decode(proj, ids_np[k], st, mult, np.array(w.rows), w.K)
        rows_of.append(idx_k)
    tabs_of = []
    for idx_k in rows_of:
        tabs = []
        for j in range(w.J):
            r = torch.from_numpy(base[j] + idx_k[:, j].astype(np.int64)).to(table.device)
            tabs.append(table.view(-1, w.D_h).index_select(0, r).double().cpu().numpy())
        tabs_of.append(tabs)
    h_of = [hs[k].reshape(w.B, 1, w.d).double().cpu().numpy() for k in range(n_steps)]
    local = np.tile(np.arange(w.B, dtype=np.int64)[:, None], (1, w.J))

    def run():
        st_r = np.full((w.B, 2), V_c_ref, np.int32)
        conv = np.zeros((w.B, 1, 3, w.d))
        for k in range(n_steps):
            _, st_r = O.hash_indices_decode(proj, ids_np[k], st_r, mult, np.array(w.rows), w.K)
            e_r = O.gather(local, tabs_of[k])
            _, _, conv = O.decode_step(e_r, h_of[k], Wk_h, Wv_h, cw_h, conv)

    sec, thr = time_oracle(run, min_s=3.0)
    return {"value": n_steps * w.B / sec, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"decode steps 0-{n_steps - 1} of all 256 sequences, fp64 on one thread "
                      f"({sec:.2f} s per run of {n_steps} steps)"}


def bench_hosttable(dev, params=8_000_000_000):
    """Host-resident table: rows gathered over PCIe from pinned host memory on
    a side stream while the compute stream runs the stand-in bf16 GEMM
    [8,192 x 2,560] x [2,560 x 10,240].  The table keeps the workload's
    16 heads x 160 dims with fewer rows per head (params) so that it fits the
    host's memory; rows stay random and far larger than any cache."""
    import torch
    from hashed_gram_conditional_engram_b200 import engram as eg
    from hashed_gram_conditional_engram_b200 import synth
    w = synth.workload("hosttable")
    per_head = params // (w.J * w.D_h)
    rows = synth.primes_at_most(per_head, w.J)
    n_el = sum(rows) * w.D_h
    host = torch.empty(n_el, dtype=torch.bfloat16, pin_memory=True)
    g = torch.Generator(device=dev)
    g.manual_seed(55)
    chunk = 1 << 29
    buf = torch.empty(chunk, dtype=torch.bfloat16, device=dev)
    for a in range(0, n_el, chunk):
        b = min(n_el, a + chunk)
        buf[: b - a].normal_(0.0, 0.02, generator=g)
        host[a:b].copy_(buf[: b - a])
    del buf
    ids_np, keys_np = synth.host_ids_keys(w)
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    keys = torch.from_numpy(keys_np).to(dev)
    proj = torch.empty(w.V, dtype=torch.int32, device=dev)
    vb = eg.engram_workspace_size(None, eg.WS_VOCAB, w.V)
    V_c = eg.engram_build_vocab_proj(keys, w.V, proj, torch.empty(vb, dtype=torch.uint8, device=dev), vb)
    cfg = eg.make_cfg(w.K, w.D_h, w.d, 1, w.V, V_c, eg.BF16, rows, mult)
    idx = torch.empty((w.B, w.T, w.J), dtype=torch.int32, device=dev)
    eg.engram_hash_indices(cfg, proj, torch.from_numpy(ids_np).to(dev), w.B, w.T, None, idx)
    e = torch.empty((w.N, w.E), dtype=torch.bfloat16, device=dev)
    idx_np = idx.cpu().numpy().reshape(w.N, w.J)
    unique_rows = int(sum(len(np.unique(idx_np[:, j])) for j in range(w.J)))
    comp = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    A = torch.randn((w.N, w.d), device=dev).to(torch.bfloat16)
    Bm = torch.randn((w.d, 4 * w.d), device=dev).to(torch.bfloat16)
    C = torch.empty((w.N, 4 * w.d), dtype=torch.bfloat16, device=dev)
    rows_bytes = w.N * w.J * w.D_h * 2
    # pinned host -> device copy peak on this machine
    src = torch.empty(1 << 30, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    ms_copy = _time_loop(lambda: dst.copy_(src, non_blocking=True), 5, 2, comp)
    h2d_peak = (1 << 30) / (ms_copy / 1e3) / 1e9
    del src, dst

    def gather():
        eg.engram_forward_hosttable(cfg, idx, host.data_ptr(), w.N, e, side, None)

    def gemm():
        torch.matmul(A, Bm, out=C)

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for _ in range(3):
        gather()
        gemm()
    torch.cuda.synchronize()
    ev[0].record(side)
    for _ in range(10):
        gather()
    ev[1].record(side)
    torch.cuda.synchronize()
    t_gather = ev[0].elapsed_time(ev[1]) / 10
    t_gemm = _time_loop(gemm, 10, 3, comp)
    # both at once: the gather on the side stream, the GEMM on the compute stream
    side.wait_stream(comp)
    torch.cuda.synchronize()
    ev[2].record(comp)
    ev[4].record(side)
    for _ in range(10):
        gather()
        gemm()
    ev[3].record(comp)
    ev[5].record(side)
    torch.cuda.synchronize()
    t_both_gemm = ev[2].elapsed_time(ev[3]) / 10
    t_both_gather = ev[4].elapsed_time(ev[5]) / 10
    if eg.engram_get_status(comp) != 0:
        raise RuntimeError("device status word set in host-table gather")
    cached = _hosttable_cached(dev, w, cfg, proj, host, idx, e, side, comp, gemm, t_gemm,
                               rows_bytes)
    # the oracle's gather of the same batch, reading the same pinned host
    # table in place (rows as bf16 bit patterns: the gather is a copy)
    from oracle import engram_oracle as O
    host_bits = host.view(torch.int16).numpy()
    starts = np.concatenate([[0], np.cumsum(rows)])
    heads = [host_bits[starts[j] * w.D_h:starts[j + 1] * w.D_h].reshape(rows[j], w.D_h)
             for j in range(w.J)]
    sec, thr = time_oracle(lambda: O.gather(idx_np, heads), min_s=2.0)
    pcie_gbs = rows_bytes / (t_gather / 1e3) / 1e9
    return {"workload": f"hosttable: 4 x 2,048 tokens, 16 heads x 160 dims, {sum(rows) * w.D_h / 1e9:.1f}B "
                        "bf16 params in pinned host memory (the 100B table does not fit the host)",
            "rows_bytes_per_batch": rows_bytes,
            "unique_rows_bytes_per_batch": unique_rows * w.D_h * 2,
            "gather_ms": t_gather,
            "pcie_gbs": rows_bytes / (t_gather / 1e3) / 1e9, "h2d_memcpy_peak_gbs": h2d_peak,
            "frac_of_h2d_peak": rows_bytes / (t_gather / 1e3) / 1e9 / h2d_peak,
            "gemm_ms_alone": t_gemm, "gemm_ms_with_gather": t_both_gemm,
            "gather_ms_with_gemm": t_both_gather,
            "gemm_slowdown": t_both_gemm / t_gemm - 1.0,
            "roofline": {"bound": "pcie", "achieved": pcie_gbs, "peak": h2d_peak, "unit": "GB/s",
                         "frac": pcie_gbs / h2d_peak, "traffic": None,
                         "bytes_per_batch": rows_bytes,
                         "peak_source": "pinned host-to-device cudaMemcpy of 1 GiB on this box"},
            "cpu_baseline": {"value": w.N / sec, "unit": "tokens/s", "cores": thr,
                             "kind": "oracle", "cpu_model": cpu_model(),
                             "rows_gbs": rows_bytes / sec / 1e9,
                             "sample": "the whole batch (8,192 tokens x 16 rows of 160 bf16) "
                                       "gathered by the oracle from the same pinned host table, "
                                       f"one thread ({sec * 1e3:.1f} ms per batch)"},
            "hbm_cache": cached}


def _hosttable_cached(dev, w, cfg, proj, host, idx, e, side, comp, gemm, t_gemm, rows_bytes,
                      history_batches=256, C=1 << 24):
    """The same batch through an HBM cache of the rows that earlier batches
    of the same distribution (history_batches x 8,192 Zipf(1.1) tokens) hit
    most: ranked on the device, copied in once, then gathered (probe, hits
    from HBM, misses over PCIe) on the side stream.  Hit rates for smaller
    caches (prefixes of the same ranking) beside it."""
    import torch
    from hashed_gram_conditional_engram_b200 import engram as eg
    from hashed_gram_conditional_engram_b200 import synth
    e_plain = e.clone()  # the uncached gather's result, to compare with
    n_hist = history_batches * w.N
    hist_ids = synth.zipf_ids(np.random.default_rng(w.seed + 1000), w.V, 1.1, n_hist,
                              perm=synth.host_ids_perm(w))
    hist_idx = torch.empty((history_batches * w.B, w.T, w.J), dtype=torch.int32, device=dev)
    eg.engram_hash_indices(cfg, proj, torch.from_numpy(hist_ids.astype(np.int32)).to(dev)
                           .reshape(history_batches * w.B, w.T), history_batches * w.B, w.T, None,
                           hist_idx)
    nb = eg.engram_workspace_size(cfg, eg.WS_HOSTCACHE_RANK, n_hist)
    rows_d = torch.empty(C, dtype=torch.int64, device=dev)
    n_out = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    eg.engram_hostcache_rank(cfg, hist_idx, n_hist, C, rows_d, n_out,
                             torch.empty(nb, dtype=torch.uint8, device=dev), nb)
    torch.cuda.synchronize()
    t_rank = time.perf_counter() - t0
    n_cached = int(n_out.item())
    cache = torch.empty((max(n_cached, 1), w.D_h), dtype=torch.bfloat16, device=dev)
    cmap = torch.empty(eg.engram_table_rows(cfg), dtype=torch.int32, device=dev)
    gb = eg.engram_workspace_size(cfg, eg.WS_HOSTCACHE_GATHER, w.N)
    gws = torch.empty(gb, dtype=torch.uint8, device=dev)
    n_miss = torch.zeros(1, dtype=torch.int32, device=dev)
    valid = int((idx >= 0).sum().item())
    hit_by_size = {}
    for c in (1 << 16, 1 << 18, 1 << 20, 1 << 22):
        if c >= n_cached:
            break
        eg.engram_hostcache_fill(cfg, host.data_ptr(), rows_d, c, cache, cmap)
        eg.engram_forward_hostcache(cfg, idx, host.data_ptr(), cache, cmap, w.N, e, n_miss, gws,
                                    gb, None, None)
        hit_by_size[str(c)] = 1.0 - int(n_miss.item()) / max(valid, 1)
    t0 = time.perf_counter()
    eg.engram_hostcache_fill(cfg, host.data_ptr(), rows_d, n_cached, cache, cmap)
    torch.cuda.synchronize()
    t_fill = time.perf_counter() - t0
    del hist_idx

    def gather():
        eg.engram_forward_hostcache(cfg, idx, host.data_ptr(), cache, cmap, w.N, e, n_miss, gws,
                                    gb, side, None)

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for _ in range(3):
        gather()
    torch.cuda.synchronize()
    if not torch.equal(e, e_plain):
        raise RuntimeError("cached gather differs from the uncached one")
    ev[0].record(side)
    for _ in range(10):
        gather()
    ev[1].record(side)
    torch.cuda.synchronize()
    t_gather = ev[0].elapsed_time(ev[1]) / 10
    side.wait_stream(comp)
    torch.cuda.synchronize()
    ev[2].record(comp)
    ev[4].record(side)
    for _ in range(10):
        gather()
        gemm()
    ev[3].record(comp)
    ev[5].record(side)
    torch.cuda.synchronize()
    t_both_gemm = ev[2].elapsed_time(ev[3]) / 10
    misses = int(n_miss.item())
    if eg.engram_get_status(comp) != 0:
        raise RuntimeError("device status word set in the cached host-table gather")
    return {"cache_rows": n_cached, "cache_bytes": n_cached * w.D_h * 2,
            "history_tokens": n_hist, "rank_s": t_rank, "fill_s": t_fill,
            "hit_rate": 1.0 - misses / max(valid, 1), "hit_rate_by_cache_rows": hit_by_size,
            "pcie_row_bytes_per_batch": misses * w.D_h * 2,
            "gather_ms": t_gather, "rows_gbs_effective": rows_bytes / (t_gather / 1e3) / 1e9,
            "gemm_ms_with_gather": t_both_gemm, "gemm_slowdown": t_both_gemm / t_gemm - 1.0}


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle, as it stands, on the host cores: each step is the first
    1,024 tokens of one sequence of this workload, end to end.  Needs no GPU:
    the table rows the sample touches are drawn on the host, row by row, with
    the workload's N(0, 0.02) statistics, outside the timed spans."""
    from hashed_gram_conditional_engram_b200 import synth
    ws_, rank = dist_init("gloo")
    if rank != 0:
        barrier()
        return None
    w = synth.workload(WORKLOAD)
    ids_np, keys_np = synth.host_ids_keys(w)
    mult = synth.hash_multipliers(synth.layer_seed(w, 0), w.J)
    rng = np.random.default_rng(w.seed + 3)
    n_tok = 1024
    dense_host = {
        "h": rng.standard_normal((n_tok, 1, w.d)),
        "Wk": rng.standard_normal((1, w.d, w.E)) * 0.02,
        "Wv": rng.standard_normal((w.d, w.E)) * 0.02,
        "conv_w": rng.standard_normal((w.d, 4)) * 0.5,
    }
    cache = {}

    def rows_fn(j, slots):
        # rows drawn on demand per (head, slot): the same row always gets the
        # same values, as a stored table would give
        out = np.empty((len(slots), w.D_h))
        for n, sl in enumerate(slots.tolist()):
            key = (j, sl)
            if key not in cache:
                cache[key] = np.random.default_rng([j, sl]).standard_normal(w.D_h) * 0.02
            out[n] = cache[key]
        return out

    times, thr = [], 1
    for i in range(args.warmup + args.steps):
        tok, sec, thr = oracle_sample(w, ids_np, keys_np, mult, rows_fn, dense_host, 1, n_tok)
        if i >= args.warmup:
            times.append(sec)
    sec = sum(times) / len(times)
    value = n_tok / sec
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": "layer27b: 27B-shaped Engram layer forward, 8 x 4,096 tokens, "
                               "d_model 2,560, orders {2,3} x 8 heads x 80 dims; oracle sample: "
                               "1,024 tokens per step", "global_batch": n_tok, "seq_len": w.T,
                   "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                         "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
                         "sample": "first 1,024 tokens of one sequence per step, end to end "
                                   "in fp64 on one thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    barrier()
    return line


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the training-step, decode and host-table measurements")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    line = run_reference(args) if args.impl == "reference" else run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
