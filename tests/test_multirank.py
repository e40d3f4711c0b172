"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

The path shards over (sequence, head) with no data exchange, so a multi-GPU
run is independent batches per rank; what needs checking is the host logic:
each rank draws a different batch, the slowest rank's time is taken (maximum
over ranks), and the whole-job rate counts every rank's units.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank time: rank 1 is the slow one
        times = bench.max_over_ranks([10.0 + 5.0 * rank, 1.0 + rank], torch.device("cpu"), dist)
        x = make_inputs(WORKLOADS["sweep_T4096"], seed=bench.rank_seed(rank), device="cpu", B=1, T=8)
        g = [torch.zeros(x["q"].shape, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(g, x["q"].float())
        distinct = not torch.equal(g[0], g[1])
        rate = bench.aggregate_rate(1000, 4, world, times[0])
        q.put((rank, times, distinct, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_aggregate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, times, distinct, rate in res:
        assert times == [15.0, 2.0]  # both ranks see the maximum over ranks
        assert distinct  # each rank drew its own batch
        assert rate == pytest.approx(1000 * 4 * 2 / 0.015)


def test_single_rank_identity():
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu"), None) == [3.0, 4.0]
    assert bench.aggregate_rate(10, 2, 1, 1000.0) == 20.0
