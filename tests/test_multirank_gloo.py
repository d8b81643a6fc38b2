"""Multi-rank host logic of the benchmark on CPU: two gloo ranks, replicas only.

Each rank times its own replica; the reported step time is the max over ranks
and the throughput counts every rank's tokens.  No tensor data crosses ranks.
"""

import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = [3.0, 5.0][rank]
        m = bench.max_over_ranks(local_ms, world)
        q.put((rank, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 5.0, 1: 5.0}


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5


def test_bandwidth_roofline_matches_the_pages_planning_numbers():
    # ExpertMesh README, hardware table: 51.2 TB/s aggregate HBM and 30-50 GB of active weights per
    # token give an ideal decode roofline of 1,024-1,707 aggregate token/s.
    import bench
    assert round(bench.hbm_roofline_tokens_per_s(51.2e12, 50e9)) == 1024
    assert round(bench.hbm_roofline_tokens_per_s(51.2e12, 30e9)) == 1707
