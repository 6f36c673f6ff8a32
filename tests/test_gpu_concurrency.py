"""Concurrent use of the library (needs a B200): calls on several streams issued from
several host threads at once give the same bytes as the same calls one after the other
(the boundary keeps no state between calls besides per-device launch configuration), and
a host thread whose first CUDA work is a call into the library (no context bound to it
yet when the tensor maps are encoded) succeeds."""
import threading

import pytest
import torch

import blockwise_adaptive_transforms_b200 as W

pytestmark = pytest.mark.gpu


def _case(seed, n, d, G):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, d, generator=g).to(torch.bfloat16).cuda()
    T = (torch.eye(G).repeat(d // G, 1, 1) + 0.1 * torch.randn(d // G, G, G, generator=g)).float().cuda()
    return x, T


JOBS = [  # (seed, rows, d_in, G, fmt): fused and CUDA-core paths, three formats
    (1, 1024, 2048, 32, "mxfp4"),
    (2, 700, 1024, 16, "nvfp4"),
    (3, 40, 4096, 32, "int4"),
    (4, 2048, 1024, 32, "mxfp4"),
    (5, 100, 2048, 16, "nvfp4"),
]


def test_threads_and_streams_at_once_equal_one_after_the_other():
    inputs = [_case(s, n, d, G) for s, n, d, G, _ in JOBS]
    expected = []
    for (x, T), job in zip(inputs, JOBS):
        expected.append(W.wush_quant_act(x, T, job[3], job[4]))
    torch.cuda.synchronize()

    results = [None] * len(JOBS)
    errors = []

    def worker(k):
        try:
            s = torch.cuda.Stream()
            x, T = inputs[k]
            outs = []
            for _ in range(4):   # several calls per thread, same stream
                outs.append(W.wush_quant_act(x, T, JOBS[k][3], JOBS[k][4], stream=s))
            s.synchronize()
            results[k] = outs
        except Exception as e:   # pragma: no cover - reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(k,)) for k in range(len(JOBS))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    for k, outs in enumerate(results):
        for o in outs:
            for a, b in zip(o, expected[k]):
                if b is not None:
                    assert torch.equal(a, b), (JOBS[k], "differs from the sequential run")


def test_first_cuda_work_of_a_fresh_thread_is_a_fused_call():
    # inputs, outputs and the stream all come from this thread, so the worker makes no
    # CUDA call of its own before the library encodes its tensor maps
    x, T = _case(6, 1024, 2048, 32)
    expected = W.wush_quant_act(x, T, 32, "mxfp4")
    codes, scales = torch.empty_like(expected[0]), torch.empty_like(expected[1])
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    errors = []

    def worker():
        try:
            W.wush_quant_act(x, T, 32, "mxfp4", codes=codes, scales=scales, stream=s)
        except Exception as e:   # pragma: no cover - reported below
            errors.append(e)

    t = threading.Thread(target=worker)
    t.start()
    t.join()
    assert not errors, errors
    s.synchronize()
    assert torch.equal(codes, expected[0]) and torch.equal(scales, expected[1])


def test_outputs_are_made_on_the_launch_stream():
    # The current stream is kept busy while the call launches on a side stream.  The
    # scale-atom buffer's zero fill must run on the launch stream, ahead of the kernel;
    # on the busy stream it would land after the kernel and wipe the scales.
    x, T = _case(7, 200, 1024, 32)
    codes, atoms = W.wush_quant_act_mx_atoms(x, T)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    torch.cuda._sleep(50_000_000)              # ~25 ms of spinning on the current stream
    c2, a2 = W.wush_quant_act_mx_atoms(x, T, stream=side)
    side.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(c2, codes) and torch.equal(a2, atoms)
    ws = W.nvfp4_workspace(stream=side)
    side.synchronize()
    assert ws.device == x.device and torch.count_nonzero(ws).item() == 0
