"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each an
independent replica with its own token batch; timing is the maximum over
ranks and the reported rate counts every rank's tokens."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist
    from hashed_gram_conditional_engram_b200 import synth
    ws, r = bench.dist_init("gloo")
    elapsed = 10.0 + 5.0 * rank                     # the slower rank sets the time
    m = bench.max_over_ranks(elapsed)
    w = synth.workload("tiny")
    w_r = synth.Workload(**{**w.__dict__, "seed": bench.rank_seed(w.seed, rank)})
    ids = synth.host_ids_keys(w_r)[0]
    bench.barrier()
    q.put((rank, ws, r, m, ids.tobytes()))
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ws0, rr0, m0, ids0), (r1, ws1, rr1, m1, ids1) = res
    assert ws0 == ws1 == 2 and (rr0, rr1) == (0, 1)
    assert m0 == m1 == 15.0
    assert ids0 != ids1                               # each replica has its own batch


def test_aggregate_rate_counts_every_rank():
    import bench
    assert bench.aggregate_rate(32768, 4, 10, 20.0) == pytest.approx(32768 * 4 * 10 / 0.02)
