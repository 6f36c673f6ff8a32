"""NVFP4 in stages (amax pass, tensor scale, quantising pass) on the device (needs a B200).

The stages must reproduce the single-call NVFP4 quantiser bit for bit; two row shards of
one batch, reduced by max between the stages (emulated on one device, without a
collective), must reproduce the full batch's codes, scales and tensor scale; an empty
shard contributes amax 0.
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W
from blockwise_adaptive_transforms_b200 import sharded

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _fused_path():
    # shards and the whole batch must take the same path (the CUDA-core path for small
    # batches rounds y differently); its own stage test is in test_gpu_small.py
    W.wush_set_small_batch_rows(0)
    yield
    W.wush_set_small_batch_rows(-1)


def _layer(n_tok, d_in):
    wl = workload("mlp_down_nvfp4_14336", n_tok=n_tok, d_in=d_in, d_out=256, n_cal=512)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 16)
    x = torch.from_numpy(np.ascontiguousarray(inp.x_bits).view(np.int16)).cuda().view(torch.bfloat16)
    return x, torch.from_numpy(b["T_wush32"]).cuda()


@pytest.mark.parametrize("n_tok,d_in", [(256, 1024), (300, 1040), (1, 4096)])
def test_stages_equal_the_single_call(n_tok, d_in):
    x, T = _layer(n_tok, d_in)
    c, s, ts = W.wush_quant_act(x, T, 16, "nvfp4")
    c2, s2, ts2 = sharded.quant_act_nvfp4_sharded(x, T)     # no process group: one rank
    torch.cuda.synchronize()
    assert torch.equal(ts, ts2) and torch.equal(c, c2) and torch.equal(s, s2)


def test_two_shards_reduced_by_max_equal_the_full_batch():
    x, T = _layer(512, 2048)
    c, s, ts = W.wush_quant_act(x, T, 16, "nvfp4")
    a0 = W.wush_quant_act_nvfp4_amax(x[:200], T)
    a1 = W.wush_quant_act_nvfp4_amax(x[200:], T)
    amax = torch.maximum(a0, a1)                              # what the all-reduce computes
    W.wush_nvfp4_scale_from_amax(amax)
    c0, s0 = W.wush_quant_act_nvfp4_with_scale(x[:200], T, amax)
    c1, s1 = W.wush_quant_act_nvfp4_with_scale(x[200:], T, amax)
    torch.cuda.synchronize()
    assert torch.equal(amax, ts)
    assert torch.equal(torch.cat([c0, c1]), c) and torch.equal(torch.cat([s0, s1]), s)
    # each shard's own scale would differ from the batch's (the exchange matters)
    assert not torch.equal(a0, a1)


def test_empty_shard_contributes_zero():
    x, T = _layer(64, 1024)
    amax = torch.full((1,), 5.0, device="cuda")
    W.wush_quant_act_nvfp4_amax(x[:0], T, amax=amax)
    torch.cuda.synchronize()
    assert amax.item() == 0.0
