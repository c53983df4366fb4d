"""The multi-GPU benchmark path runs independent replicas (weak scaling):
the only collective reduces the measurements -- max of device time, sum of
work.  Checked here with two gloo ranks on the CPU."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.aggregate(1.0 + rank, 100.0 * (rank + 1), 10.0 * (rank + 1), world, torch.device("cpu"))
    q.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_replicas_report_slowest_time_and_total_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == (2.0, 300.0, 30.0)


def test_single_rank_passes_through():
    import bench
    assert bench.aggregate(3.0, 7.0, 2.0, 1, None) == (3.0, 7.0, 2.0)
