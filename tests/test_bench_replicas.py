"""The bench's multi-GPU path runs independent replicas (the MoE branch is
independent per token; there is no collective on the data path).  The host
logic around the replicas -- slowest-replica time by an all-reduce MAX over
ranks, whole-job throughput, disjoint input pools -- is checked here on the
CPU with two `gloo` ranks."""
import datetime
import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r's timed region took 100 + 7 r ms over 50 steps of 64 tokens
        total_ms = bench.max_over_ranks(100.0 + 7.0 * rank, world, "cpu")
        q.put((rank, total_ms, bench.job_rate(64, world, 50, total_ms)))
    finally:
        dist.destroy_process_group()


def test_slowest_replica_time_and_job_rate_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    for rank, total_ms, rate in got:
        assert total_ms == 107.0                      # every rank sees the slowest replica
        assert abs(rate - 2 * 64 * 50 / 0.107) < 1e-6  # all ranks' tokens over that time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.job_rate(1, 1, 10, 1000.0) == 10.0


def test_replica_input_pools_are_disjoint():
    n_pool = 64
    pools = [{bench.replica_x_seed(r, n_pool, i) for i in range(n_pool)} for r in range(8)]
    assert sum(len(p) for p in pools) == len(set().union(*pools)) == 8 * n_pool
