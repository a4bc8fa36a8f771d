"""Host logic of the multi-GPU bench (independent replicas, max-over-ranks timing), run as two
gloo ranks on the CPU."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 17.25][rank]  # this rank's device time for K steps
        m = bench.max_over_ranks(ms, world, "cpu")
        v = bench.aggregate_throughput(4096 * 10, world, m / 1e3)
        bench.barrier(world)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_timing_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in got:
        assert m == 17.25  # the slowest rank's time
        assert abs(v - 2 * 4096 * 10 / 17.25e-3) < 1e-6
