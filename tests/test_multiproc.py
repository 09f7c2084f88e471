"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
the replicas' timings are reduced by max over ranks and the whole-job
throughput counts every rank's tokens. The GPU path itself shards by batch
with no data-path collective, so this is the only cross-rank logic."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # rank r measured (10 + r) ms in total and (3 + 2r, 7 - r) ms per run
    m = bench.allreduce_max([10.0 + rank, 3.0 + 2 * rank, 7.0 - rank], device="cpu")
    v = bench.job_throughput(1000, 2, world, m[0])
    out.put((rank, m, v))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_reduction_and_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v in res:
        assert m == [11.0, 5.0, 7.0]                  # max over ranks, element-wise
        assert abs(v - 2 * 1000 * 2 / 0.011) < 1e-6  # all ranks' tokens / slowest time


def test_single_process_reduction_is_identity():
    import bench
    assert bench.allreduce_max([1.0, 2.5], device="cpu") == [1.0, 2.5]
    assert bench.job_throughput(64, 3, 1, 1000.0) == 192.0
