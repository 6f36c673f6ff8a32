"""GPTQ-WUSH host pipeline (torch, float64 on the GPU) vs the fp64 oracle, and its use
with the online kernels (needs a B200).  Section: paper-graph-ui analysis, 3.4.6 "GPTQ
Integration (Algorithm 1)", re-derived as documented in the oracle (reading R12).
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W
from blockwise_adaptive_transforms_b200 import gptq_wush as GW

pytestmark = pytest.mark.gpu

LAYERS = [("tiny_mxfp4", {}), ("attn_mxfp4_4096", dict(n_tok=256, d_in=512, d_out=256, n_cal=1024))]


def dev_x(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("gptq", [False, True])
@pytest.mark.parametrize("fmt", ["mxfp4", "int4"])
@pytest.mark.parametrize("name,over", LAYERS, ids=[l[0] for l in LAYERS])
def test_pipeline_matches_oracle(name, over, fmt, gptq):
    wl = workload(name, **over)
    inp = make_inputs(wl)
    ref = O.gptq_wush(inp.w, inp.xcal_bits, 32, fmt, gptq=gptq)
    got = GW.gptq_wush(torch.from_numpy(inp.w).cuda(), dev_x(inp.xcal_bits), 32, fmt, gptq=gptq)
    T = got["T_act64"].cpu().numpy()
    assert np.max(np.abs(T - ref["T_act"])) <= 1e-8 * np.max(np.abs(ref["T_act"]))
    cg = O.unpack_nibbles(got["codes"].cpu().numpy())
    co = O.unpack_nibbles(ref["codes"])
    assert np.mean(cg != co) <= 1e-3
    sg, so = got["scales"].cpu().numpy(), ref["scales"]
    same = (sg == so) if fmt == "mxfp4" else (np.abs(sg.astype(np.float64) - so) <= 2.0 ** -20 * np.abs(so))
    assert np.mean(~same) <= 1e-3


@pytest.mark.parametrize("fmt", ["mxfp4", "int4"])
def test_pipeline_with_the_online_kernels(fmt):
    """Activations through wush_quant_act with the pipeline's T_X, weights dequantised by
    wush_dequant: the layer loss matches the oracle's and error feedback beats RTN."""
    wl = workload("attn_mxfp4_4096", n_tok=256, d_in=512, d_out=256, n_cal=1024)
    inp = make_inputs(wl)
    w = torch.from_numpy(inp.w).cuda()
    xcal = dev_x(inp.xcal_bits)
    losses = {}
    for gq in (False, True):
        r = GW.gptq_wush(w, xcal, 32, fmt, gptq=gq)
        cx, sx, tx = W.wush_quant_act(xcal, r["T_act"], 32, fmt)
        xq = W.wush_dequant(cx, sx, tx, 32, fmt).double()
        wq = W.wush_dequant(r["codes"], r["scales"], None, 32, fmt).double()
        ref = w.double() @ xcal.double().T
        err = ref - wq @ xq.T
        losses[gq] = float((err * err).mean())
        o = O.gptq_wush(inp.w, inp.xcal_bits, 32, fmt, gptq=gq)
        lo = O.layer_loss_prequantised(o["Wq"], inp.w, inp.xcal_bits, o["T_act"].astype(np.float32), fmt, 32)
        assert abs(losses[gq] - lo) <= 0.02 * lo, (gq, losses[gq], lo)
    assert losses[True] < losses[False]


def test_gptq_weights_feed_the_fp4_gemm():
    wl = workload("attn_mxfp4_4096", n_tok=256, d_in=512, d_out=256, n_cal=1024)
    inp = make_inputs(wl)
    r = GW.gptq_wush(torch.from_numpy(inp.w).cuda(), dev_x(inp.xcal_bits), 32, "mxfp4")
    x = dev_x(inp.x_bits)
    cx, ax = W.wush_quant_act_mx_atoms(x, r["T_act"])
    d = W.wush_gemm_mxfp4(cx, ax, r["codes"], W.wush_mx_scales_to_atoms(r["scales"]))
    sx = W.wush_quant_act(x, r["T_act"], 32, "mxfp4")[1]
    torch.cuda.synchronize()
    ref = O.gemm_mx(cx.cpu().numpy(), sx.cpu().numpy(), r["codes"].cpu().numpy(), r["scales"].cpu().numpy())
    assert np.allclose(d.float().cpu().numpy(), ref, rtol=2 ** -7, atol=1e-3 * np.max(np.abs(ref)))
