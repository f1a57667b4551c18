"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

Every rank runs its own sequence (weak scaling, no collective on the data path); the
only exchange is the timing reduction: whole-job throughput is all ranks' tokens over
the slowest rank's time.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms_local = [40.0, 55.0][rank]
    ms_max, value = bench.aggregate_max(ms_local, 32768 * 10, world, device="cpu")
    q.put((rank, ms_max, value))
    dist.barrier()
    dist.destroy_process_group()


def test_weak_scaling_aggregate_is_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, value in res:
        assert ms_max == 55.0
        assert abs(value - 2 * 32768 * 10 / 0.055) < 1e-6 * value


def test_single_rank_aggregate_needs_no_process_group():
    import bench
    ms_max, value = bench.aggregate_max(20.0, 1000, 1, device="cpu")
    assert ms_max == 20.0 and abs(value - 50000.0) < 1e-9
