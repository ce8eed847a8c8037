"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the
job time is the slowest rank's, the throughput counts every rank's bytes,
and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    t = bench.max_over_ranks(world, ms)
    v = bench.job_throughput(1e9, 10, world, t)
    out[rank] = (t, v)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_job_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0
    # 2 ranks x 10 steps x 1 GB in 15 ms
    assert abs(out[0][1] - 2 * 10 * 1.0 / 0.015) < 1e-6


def test_reference_arm_runs_on_rank0_only(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        warmup, steps, steps_given = 3, 1, True
    bench.run_reference(A())
    assert capsys.readouterr().out == ""
