"""The benchmark's multi-rank bookkeeping on CPU with gloo (world size 2): the job time is
the slowest rank's, throughput is weak-scaled over ranks, and the reference arm runs on
rank 0 only."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    elapsed = 1.0 + rank          # rank 1 is slower
    out[rank] = bench.max_over_ranks(elapsed)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1] == 2.0
    import bench
    # two ranks, each 10 steps of 1e9 bytes in 2 s -> 10 GB/s for the job
    assert bench.job_throughput(2, 10, 10 ** 9, 2.0) == pytest.approx(10.0)


def test_single_process_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_is_silent_on_nonzero_ranks(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 1, 2
    bench.run_reference(A())
    assert capsys.readouterr().out == ""
