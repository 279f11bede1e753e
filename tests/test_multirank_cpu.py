"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each
rank serves its own request, the timed region's maximum over ranks is used,
and the whole-job throughput counts every rank's bytes."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    local = [2.0 + rank, 5.0 - 3 * rank, 1.5]          # rank 0: [2, 5, 1.5]; rank 1: [3, 2, 1.5]
    mx = bench.max_over_ranks(local, dist)
    dist.barrier()
    q.put((rank, mx, bench.job_throughput(world, 1e9, mx[0])))
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gbs in out:
        assert mx == [3.0, 5.0, 1.5]                    # every rank sees the same maxima
        assert gbs == pytest.approx(2 * 1e9 / 3e-3 / 1e9)   # 2 ranks x 1 GB in 3 ms


def test_single_process_reduction_is_identity():
    import bench
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
    assert bench.job_throughput(1, 26e9, 4.0) == pytest.approx(6500.0)
