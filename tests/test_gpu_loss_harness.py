"""Layerwise-loss harness and the dequantisation kernel vs the fp64 oracle (needs a B200).

The loss is the pages' normalised Frobenius layer loss (paper-graph-ui analysis,
section 3.4.1, Eq. (5); section 5 "Per-Layer Quantization Loss (Table 1)").  Transforms
fed to both sides come from the oracle's builder, so no oracle input comes from the
CUDA path.
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W
from blockwise_adaptive_transforms_b200 import loss_harness as LH

pytestmark = pytest.mark.gpu

FORMATS = [("mxfp4", 32), ("nvfp4", 16), ("int4", 32), ("int4", 16)]


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


@pytest.mark.parametrize("fmt,G", FORMATS)
def test_dequant_is_the_exact_product_rounded_once(fmt, G):
    wl = workload("attn_mxfp4_4096", n_tok=257, d_in=416, n_cal=64, d_out=64)
    inp = make_inputs(wl, need_w=False, need_cal=False)
    C = wl.d_in // G
    T = dev_f32(np.stack([np.eye(G)] * C))
    c, s, ts = W.wush_quant_act(dev_bf16(inp.x_bits), T, G, fmt)
    out = W.wush_dequant(c, s, ts, G, fmt)
    torch.cuda.synchronize()
    ts_v = None if ts is None else float(ts.cpu().numpy()[0])
    expect = O.dequant(O.unpack_nibbles(c.cpu().numpy()), s.cpu().numpy(), fmt, G, ts_v).astype(np.float32)
    got = out.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), expect.view(np.uint32)) or np.array_equal(got, expect)


@pytest.mark.parametrize("fmt,G", [("mxfp4", 32), ("nvfp4", 16), ("int4", 32)])
def test_harness_loss_matches_oracle(fmt, G):
    wl = workload("tiny_mxfp4")
    inp = make_inputs(wl)
    C = wl.d_in // G
    b = O.build_transforms(inp.w, inp.xcal_bits, G)
    bw = O.build_transforms(inp.w, inp.xcal_bits, G, use_hadamard=False)
    I = np.stack([np.eye(G)] * C).astype(np.float32)
    H = np.stack([O.sylvester_hadamard(G)] * C).astype(np.float32)
    cases = {"I": (I, I), "H": (H, H), "WUS": (bw["T_wush32"], bw["T_xvsh32"]),
             "WUSH": (b["T_wush32"], b["T_xvsh32"])}
    w = dev_f32(inp.w)
    x = dev_bf16(inp.xcal_bits)
    for kind, (Ta, Tw) in cases.items():
        got = LH.layer_loss(w, x, dev_f32(Ta), dev_f32(Tw), G, fmt)
        ref = O.layer_loss(inp.w, inp.xcal_bits, Tw, Ta, fmt, G)
        assert abs(got - ref) <= 1e-2 * ref, (kind, got, ref)


def test_loss_table_orders_the_transforms_as_the_pages_report():
    """On the synthetic layer with outlier channels: WUSH has the lowest loss for MXFP4
    and INT4, and the data-dependent transforms (WUS, WUSH) beat I and H for NVFP4."""
    res = LH.loss_table("tiny_mxfp4", rand_runs=3)
    for fmt in ("mxfp4", "int4"):
        row = res["loss"][fmt]
        assert row["WUSH"] == min(row.values()), (fmt, row)
    row = res["loss"]["nvfp4"]
    assert max(row["WUS"], row["WUSH"]) < min(row["I"], row["H"]), row
