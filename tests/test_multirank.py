"""Multi-process (gloo, world size 2, CPU) checks of the data-parallel benchmark plumbing: every
rank gets its own seeded sequence of the same shapes, the step time is the maximum over ranks,
and a rank that fails before joining is reported by the others' rendezvous timeout instead of a
hang."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from sparse_attention_compressor_b200 import workloads as W
    bench.init_dist(world, "gloo")
    wl = bench.rank_workload(W.WORKLOADS["tiny_csa_f32"], rank)
    x = W.prefill_inputs(wl, with_queries=False)
    bench.barrier()
    t = bench.max_over_ranks(10.0 + rank)
    out.put((rank, wl.seed, float(x["kv"].sum()), t))
    torch.distributed.destroy_process_group()


def test_ranks_get_distinct_sequences_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    seeds = [r[1] for r in res]
    sums = [r[2] for r in res]
    assert seeds[0] != seeds[1] and sums[0] != sums[1]
    assert all(r[3] == 11.0 for r in res)


def _lonely(port, out):
    sys.path.insert(0, ROOT)
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="2")
    try:
        torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=3))
        torch.distributed.barrier()
        out.put("joined")
    except Exception as e:  # the peer never joins: rendezvous / barrier times out
        out.put(type(e).__name__)


def test_missing_rank_times_out_instead_of_hanging():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    p = ctx.Process(target=_lonely, args=(_free_port(), q))
    p.start()
    p.join(timeout=90)
    if p.is_alive():
        p.kill()
        pytest.fail("rank 0 hung waiting for a missing peer")
    assert q.get() != "joined"
