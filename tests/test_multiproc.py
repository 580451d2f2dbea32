"""The N > 1 path of bench.py on CPU: two gloo ranks (replicas, no data-path
collective) agree on the slowest rank's step time and on the whole-job value."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [2.0, 3.5][rank]
        bench.barrier(world)
        slowest = bench.max_over_ranks(world, local_ms, device="cpu")
        value = bench.replica_throughput(world, 1.0e12, slowest)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_slowest_time_and_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for _, slowest, value in res:
        assert slowest == 3.5
        # 2 replicas x 1 TFLOP each in 3.5 ms
        assert abs(value - 2 * 1.0e12 / 3.5e-3 / 1e12) < 1e-9


def test_single_rank_is_identity():
    assert bench.max_over_ranks(1, 4.2) == 4.2
    assert abs(bench.replica_throughput(1, 2.0e12, 4.0) - 500.0) < 1e-9
