"""The CUDA-core path for decode-sized activation batches vs the fp64 oracle (needs a B200).

Batches of at most `wush_set_small_batch_rows` rows (default 64 MXFP4, 256 otherwise) skip the fused
tensor-core kernel.  Each case checks rule 1 (the oracle's quantiser on the kernel's own
fp32 y gives the kernel's codes and scales bit for bit), that y is the fp32-FMA transform
(within G * 2^-23 of |T_i||x| of the float64 product), rule 2 end to end, and the same
two rules for the fused kernel forced onto the same batch (the two paths' y differ by
rounding, so for NVFP4 even their tensor scales may differ: each is held to the oracle).
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W
from parity_rules import assert_bit_exact, assert_end_to_end

pytestmark = pytest.mark.gpu

CASES = [  # workload, fmt, G, d_in (ragged block counts)
    ("attn_mxfp4_4096", "mxfp4", 32, 1056),
    ("mlp_down_nvfp4_14336", "nvfp4", 16, 1040),
    ("int4_sweep_4096", "int4", 32, 1056),
    ("int4_sweep_4096", "int4", 16, 1040),
]


@pytest.fixture(autouse=True)
def _default_threshold():
    W.wush_set_small_batch_rows(-1)
    yield
    W.wush_set_small_batch_rows(-1)


def _data(name, fmt, G, d_in, n_tok):
    over = dict(n_tok=n_tok, d_in=d_in, d_out=2048, n_cal=512)   # transforms from a realistically wide layer
    if name == "int4_sweep_4096":
        over["G"] = G
    wl = workload(name, **over)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, G)
    x = torch.from_numpy(np.ascontiguousarray(inp.x_bits).view(np.int16)).cuda().view(torch.bfloat16)
    return inp, b, x, torch.from_numpy(b["T_wush32"]).cuda()


def _ts(ts):
    return None if ts is None else float(ts.item())


@pytest.mark.parametrize("n_tok", [1, 7, 64])
@pytest.mark.parametrize("name,fmt,G,d_in", CASES)
def test_small_batches_against_the_oracle(name, fmt, G, d_in, n_tok):
    inp, b, x, T = _data(name, fmt, G, d_in, n_tok)
    c, s, ts, y = W.wush_quant_act_debug(x, T, G, fmt)
    c2, s2, ts2 = W.wush_quant_act(x, T, G, fmt)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    assert torch.equal(c, c2) and torch.equal(s, s2)
    assert_bit_exact(c.cpu().numpy(), s.cpu().numpy(), _ts(ts), y.cpu().numpy(), fmt, G)
    x64 = O.bf16_to_f64(inp.x_bits)
    y_ref = O.block_transform(x64, b["T_wush32"].astype(np.float64))
    bound = O.block_transform(np.abs(x64), np.abs(b["T_wush32"].astype(np.float64)))
    assert np.all(np.abs(y.cpu().numpy() - y_ref) <= G * 2.0 ** -23 * bound + 1e-300)
    assert_end_to_end(c.cpu().numpy(), s.cpu().numpy(), _ts(ts), y_ref, fmt, G)

    # the fused tensor-core kernel on the same batch
    W.wush_set_small_batch_rows(0)
    cf, sf, tsf, yf = W.wush_quant_act_debug(x, T, G, fmt)
    torch.cuda.synchronize()
    assert_bit_exact(cf.cpu().numpy(), sf.cpu().numpy(), _ts(tsf), yf.cpu().numpy(), fmt, G)
    assert_end_to_end(cf.cpu().numpy(), sf.cpu().numpy(), _ts(tsf), y_ref, fmt, G)


def test_shared_matrix_small_batch_equals_per_block_copies():
    inp, b, x, _ = _data("attn_mxfp4_4096", "mxfp4", 32, 1024, 5)
    H = W.wush_hadamard(32)
    c, s, _ = W.wush_quant_act_shared(x, H, 32, "mxfp4")
    c2, s2, _ = W.wush_quant_act(x, H.repeat(32, 1, 1).contiguous(), 32, "mxfp4")
    torch.cuda.synchronize()
    assert torch.equal(c, c2) and torch.equal(s, s2)


def test_nvfp4_stages_take_the_small_path_too():
    inp, b, x, T = _data("mlp_down_nvfp4_14336", "nvfp4", 16, 1024, 40)
    c, s, ts = W.wush_quant_act(x, T, 16, "nvfp4")
    a0 = W.wush_quant_act_nvfp4_amax(x[:17], T)
    a1 = W.wush_quant_act_nvfp4_amax(x[17:], T)
    amax = torch.maximum(a0, a1)
    W.wush_nvfp4_scale_from_amax(amax)
    c0, s0 = W.wush_quant_act_nvfp4_with_scale(x[:17], T, amax)
    c1, s1 = W.wush_quant_act_nvfp4_with_scale(x[17:], T, amax)
    torch.cuda.synchronize()
    assert torch.equal(amax, ts)
    assert torch.equal(torch.cat([c0, c1]), c) and torch.equal(torch.cat([s0, s1]), s)


def test_threshold_setter_rejects_huge_values():
    with pytest.raises(W.WushError):
        W.wush_set_small_batch_rows(1 << 21)


@pytest.mark.parametrize("fmt,n_tok,d_in", [("mxfp4", 40, 1056), ("nvfp4", 200, 1040)])
def test_small_batches_write_scale_atoms(fmt, n_tok, d_in):
    """The scale-atom quantisers take the same path as the row-major ones for the same
    batch: same codes, and the atoms hold the row-major scales in the atom layout."""
    G = 32 if fmt == "mxfp4" else 16
    name = "attn_mxfp4_4096" if fmt == "mxfp4" else "mlp_down_nvfp4_14336"
    inp, b, x, T = _data(name, fmt, G, d_in, n_tok)
    c, s, ts = W.wush_quant_act(x, T, G, fmt)
    if fmt == "mxfp4":
        ca, at = W.wush_quant_act_mx_atoms(x, T)
    else:
        ca, at, tsa = W.wush_quant_act_nv_atoms(x, T)
    torch.cuda.synchronize()
    assert torch.equal(c, ca)
    if fmt == "nvfp4":
        assert torch.equal(ts, tsa)
    assert np.array_equal(at.cpu().numpy(), O.scale_atoms(s.cpu().numpy()))


def test_narrow_layer_rule2_statistic():
    """Rule 2 on a deliberately narrow layer (transforms from 128 output channels), the
    case where a single legitimate one-step flip of a top-magnitude NVFP4 code moves the
    relative Frobenius error past 2e-3.  The flip budget and the one-step bound still hold;
    the Frobenius figure is recorded (printed) and held to the 4e-3 that one such flip in
    this batch can produce, not to 2e-3 (the other tests build their transforms from
    realistically wide layers)."""
    from parity_rules import end_to_end_report
    wl = workload("mlp_down_nvfp4_14336", n_tok=64, d_in=1040, d_out=128, n_cal=512)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 16)
    x = torch.from_numpy(np.ascontiguousarray(inp.x_bits).view(np.int16)).cuda().view(torch.bfloat16)
    T = torch.from_numpy(b["T_wush32"]).cuda()
    W.wush_set_small_batch_rows(0)                 # the tensor-core kernel (hi/lo split)
    c, s, ts = W.wush_quant_act(x, T, 16, "nvfp4")
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    y_ref = O.block_transform(O.bf16_to_f64(inp.x_bits), b["T_wush32"].astype(np.float64))
    rel, frac, nsd, mx = end_to_end_report(c.cpu().numpy(), s.cpu().numpy(), ts.item(), y_ref, "nvfp4", 16)
    print(f"narrow layer (128 outputs), NVFP4 64 x 1040: rel-Frobenius {rel:.3e}, "
          f"codes differing {frac:.3e}, groups with a different scale {nsd}, max steps {mx}")
    assert mx <= 1 and frac <= 1e-3
    assert rel <= 4e-3
