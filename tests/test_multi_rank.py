"""The replicas-only multi-GPU path of the benchmark, exercised on the CPU with
two gloo ranks: each rank reports its own time, all ranks agree on the
slowest one, and the job throughput counts every rank's batch at that pace."""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    mine = 10.0 + 5.0 * rank           # rank 1 is the slow one
    got = bench.max_over_ranks(mine, torch.device("cpu"))
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_time_and_job_throughput():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 15.0, 1: 15.0}
    import bench
    # 2 ranks x 16 sequences per 15 ms / 1000 steps
    assert bench.job_tokens_per_s(2, 16, 15.0 / 1000) == pytest.approx(2 * 16 / 15e-6)
