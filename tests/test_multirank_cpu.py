"""The benchmark's multi-rank logic on CPU: two gloo ranks on 127.0.0.1.

The decode path shards over independent sequences (replicas, no data-path
collective); what crosses ranks is only the timing reduction: the slowest
rank's time and the sum of all ranks' query tokens."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import sys

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from compressed_sparse_kv_04_b200 import configs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        barrier, rmax, rsum = bench.make_reducers(world, torch.device("cpu"))
        barrier()
        # Rank r "took" 10 + 5r ms for its 8 sequences x 100 steps.
        value, t = bench.aggregate(8 * 100, 10.0 + 5.0 * rank, world, rmax, rsum)
        w = bench.workload_for_rank(configs.CSA_128K, rank)
        barrier()
        q.put((rank, value, t, w.seed, w.name, w.B))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_aggregate_and_independent_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=100) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    # Whole-job throughput: all ranks' tokens over the slowest rank's time.
    for _, value, t, _, _, _ in res:
        assert t == 15.0
        assert value == pytest.approx(2 * 800 / 0.015)
    # Same workload shape on every rank, independent inputs (own seed).
    assert res[0][4] == res[1][4] and res[0][5] == res[1][5]
    assert res[0][3] != res[1][3]


def test_single_rank_reducers_are_identity():
    import torch

    import bench
    barrier, rmax, rsum = bench.make_reducers(1, torch.device("cpu"))
    barrier()
    assert rmax(3.5) == 3.5 and rsum(2.0) == 2.0
    assert bench.aggregate(800, 10.0, 1, rmax, rsum) == (80000.0, 10.0)
