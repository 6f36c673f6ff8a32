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


# ---------------------------------------------------------------- sharded NVFP4 (host logic)
# The device stages are replaced by host stand-ins built on the oracle, so the test checks
# the rank logic alone: one max all-reduce between the amax pass and the quantising pass,
# the same tensor scale on every rank, and each rank's codes for its own rows.

def _nv_fakes():
    import numpy as np
    from oracle import wush_oracle as O

    def y_of(x, T):
        return O.block_transform(O.bf16_to_f64(x.view(torch.int16).numpy().view(np.uint16)), T.numpy())

    def amax(x, T, stream=None):
        y = y_of(x, T)
        return torch.tensor([float(O.fl32(np.max(np.abs(y))) if y.size else 0.0)], dtype=torch.float32)

    def scale(a, stream=None):
        a.copy_(torch.tensor([O.nvfp4_tensor_scale(float(a.item()))], dtype=torch.float32))
        return a

    def quantise(x, T, ts, codes=None, scales=None, stream=None):
        c, s, _ = O.quant_nvfp4(y_of(x, T), float(ts.item()))
        return torch.from_numpy(O.pack_nibbles(c)), torch.from_numpy(s)
    return {"amax": amax, "scale": scale, "quantise": quantise}


def _nv_inputs():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(48, 64, generator=g)
    x[40:] *= 9.0                               # the largest rows live on rank 1
    T = (torch.eye(16) + 0.2 * torch.randn(4, 16, 16, generator=g)).to(torch.float32)
    return x.to(torch.bfloat16), T


def _nv_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from blockwise_adaptive_transforms_b200 import sharded
    sharded._stages.update(_nv_fakes())
    x, T = _nv_inputs()
    rows = x[rank * 24:(rank + 1) * 24]
    codes, scales, ts = sharded.quant_act_nvfp4_sharded(rows, T)
    out[rank] = (float(ts.item()), codes.numpy().tobytes(), scales.numpy().tobytes())
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_nvfp4_reduces_the_tensor_scale_across_ranks():
    import numpy as np
    from oracle import wush_oracle as O
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_nv_worker, args=(world, port, out), nprocs=world, join=True)
    x, T = _nv_inputs()
    y = O.block_transform(O.bf16_to_f64(x.view(torch.int16).numpy().view(np.uint16)), T.numpy())
    # the whole batch on one device; the amax travels as fp32 (as on the device)
    s_t = O.nvfp4_tensor_scale(float(np.float32(np.max(np.abs(y)))))
    codes, scales, _ = O.quant_nvfp4(y, s_t)
    assert out[0][0] == out[1][0] == np.float32(s_t)
    for r in range(world):
        assert out[r][1] == O.pack_nibbles(codes[r * 24:(r + 1) * 24]).tobytes()
        assert out[r][2] == scales[r * 24:(r + 1) * 24].tobytes()
    # without the exchange rank 0 would pick a smaller scale from its own rows
    assert O.nvfp4_tensor_scale(float(np.float32(np.max(np.abs(y[:24]))))) < s_t
