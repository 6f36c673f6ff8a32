"""Chains of calls captured in a CUDA graph (needs a B200).

The kernels launch with programmatic stream serialisation, and inside a graph that
becomes programmatic edges. Each step's input buffer is refilled by a torch copy before
the quantisers read it. The NVFP4 calls then run their four dependent launches on the
CUDA-core path and on the fused path. INT4 runs on the CUDA-core path, and the MXFP4
quantiser feeds the FP4 GEMM. Every replayed output must equal the same call made
eagerly on the same input.
"""
import pytest
import torch

import blockwise_adaptive_transforms_b200 as W

pytestmark = pytest.mark.gpu

D_IN = 1024
STEPS = 3


def _T(G, seed):
    g = torch.Generator().manual_seed(seed)
    C = D_IN // G
    return (torch.eye(G).repeat(C, 1, 1) + 0.1 * torch.randn(C, G, G, generator=g)).float().cuda()


def test_replayed_chain_equals_eager_calls():
    g = torch.Generator().manual_seed(11)
    srcs = [torch.randn(512, D_IN, generator=g).mul(1.0 + k).to(torch.bfloat16).cuda() for k in range(STEPS)]
    T16, T32 = _T(16, 1), _T(32, 2)
    w = torch.randn(256, D_IN, generator=g).float().cuda()
    wc, wa = W.wush_quant_weight_mx_atoms(w, T32)

    def step(x, outs=None):
        o = outs or {}
        r = {}
        r["nv_small"] = W.wush_quant_act(x[:64], T16, 16, "nvfp4", *o.get("nv_small", (None, None, None)))
        r["nv_fused"] = W.wush_quant_act(x, T16, 16, "nvfp4", *o.get("nv_fused", (None, None, None)))
        r["int4"] = W.wush_quant_act(x[:16], T32, 32, "int4", *o.get("int4", (None, None, None)))
        ac, aa = W.wush_quant_act_mx_atoms(x[:256], T32, *o.get("atoms", (None, None)))
        r["atoms"] = (ac, aa)
        r["gemm"] = (W.wush_gemm_mxfp4(ac, aa, wc, wa, out=o.get("gemm", (None,))[0]),)
        return r

    torch.cuda.synchronize()
    W.wush_set_small_batch_rows(-1)            # the per-format defaults: 64 and 16 rows small, 512 fused
    expected = [step(s) for s in srcs]
    torch.cuda.synchronize()

    xbuf = torch.empty_like(srcs[0])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        outs = [step(srcs[0]) for _ in range(STEPS)]   # output buffers, made on the capture stream
        side.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for k in range(STEPS):
                xbuf.copy_(srcs[k])
                step(xbuf, outs[k])
    for o in outs:                             # replay must overwrite every output
        for v in o.values():
            for t in v:
                if t is not None:
                    t.zero_()
    torch.cuda.synchronize()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    for k in range(STEPS):
        for name, v in expected[k].items():
            for a, b in zip(outs[k][name], v):
                if b is not None:
                    assert torch.equal(a, b), (k, name)
