"""CUDA path vs the independent fp64 oracle (needs a B200).

Every case: inputs from the seeded workload generator, transforms from the oracle's
builder (so no oracle input comes from the CUDA path), then
  rule 1: oracle quantiser on the kernel's own fp32 y == kernel codes/scales, bit for bit;
  rule 2: kernel output vs oracle float64 path: rel. Frobenius <= 2e-3, <= 0.1 % codes
          differ, each by one grid step.
Shapes span several 128-row x 128-channel tiles with ragged row and channel tails.
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import bf16_bits_from_f64, make_inputs, workload
import blockwise_adaptive_transforms_b200 as W
from parity_rules import assert_bit_exact, assert_end_to_end, canon_codes

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host(t):
    return None if t is None else t.cpu().numpy()


def ts_value(ts):
    return None if ts is None else float(ts.cpu().numpy()[0])


def assert_within_split_bound(y_gpu, y_ref, x64, T32, rel):
    """Elementwise |y_gpu - y| <= rel * (|T_i| |x|) per block.

    The kernel multiplies with T = T_hi + T_lo in bf16 (|T - T_hi - T_lo| <= 2^-17 |T|)
    and, for fp32 inputs, x = x_hi + x_lo (the dropped x_lo T_lo term is <= 2^-16 |x||T|),
    accumulating in fp32 (G terms, <= G * 2^-24 relative to |T||x|); rel = 2^-15 for
    bf16 activations and 2^-14 for fp32 weights cover these with margin."""
    bound = O.block_transform(np.abs(x64), np.abs(T32.astype(np.float64)))
    err = np.abs(np.asarray(y_gpu, np.float64) - y_ref)
    worst = np.max(err / (bound + 1e-300))
    assert worst <= rel, f"transform error {worst:.3e} of |T||x| exceeds {rel:.3e}"


def assert_device_clean():
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"


CASES = [
    ("tiny_mxfp4", {}, "mxfp4", 32),
    ("attn_mxfp4_4096", dict(n_tok=300, d_in=416, d_out=256, n_cal=512), "mxfp4", 32),
    ("mlp_down_nvfp4_14336", dict(n_tok=300, d_in=400, d_out=256, n_cal=512, n_outliers=4), "nvfp4", 16),
    ("int4_sweep_4096", dict(n_tok=300, d_in=416, d_out=256, n_cal=512), "int4", 32),
    ("int4_sweep_4096", dict(n_tok=300, d_in=400, G=16, d_out=256, n_cal=512), "int4", 16),
]
IDS = [f"{c[0]}-{c[2]}{c[3]}-{c[1].get('n_tok', 'full')}x{c[1].get('d_in', 'full')}" for c in CASES]

_CACHE = {}


def case_data(name, over):
    key = (name, tuple(sorted(over.items())))
    if key not in _CACHE:
        wl = workload(name, **over)
        inp = make_inputs(wl)
        b = O.build_transforms(inp.w, inp.xcal_bits, wl.G)
        _CACHE[key] = (wl, inp, b)
    return _CACHE[key]


@pytest.mark.parametrize("name,over,fmt,G", CASES, ids=IDS)
def test_act_bit_exact_given_kernel_y(name, over, fmt, G):
    wl, inp, b = case_data(name, over)
    x = dev_bf16(inp.x_bits)
    T = dev_f32(b["T_wush32"])
    c, s, ts, y = W.wush_quant_act_debug(x, T, G, fmt)
    torch.cuda.synchronize()
    assert_device_clean()
    assert_bit_exact(host(c), host(s), ts_value(ts), host(y), fmt, G)
    # the kernel's fp32 y agrees with the float64 transform within the hi+lo split bound
    x64 = O.bf16_to_f64(inp.x_bits)
    y_ref = O.block_transform(x64, b["T_wush32"].astype(np.float64))
    assert_within_split_bound(host(y), y_ref, x64, b["T_wush32"], 2.0 ** -15)


@pytest.mark.parametrize("name,over,fmt,G", CASES, ids=IDS)
def test_act_end_to_end_and_repeatable(name, over, fmt, G):
    wl, inp, b = case_data(name, over)
    x = dev_bf16(inp.x_bits)
    T = dev_f32(b["T_wush32"])
    outs = [W.wush_quant_act(x, T, G, fmt) for _ in range(3)]
    torch.cuda.synchronize()
    assert_device_clean()
    c0, s0, ts0 = (host(t) for t in outs[0])
    for c, s, ts in outs[1:]:                  # nondeterminism would reveal a race
        assert np.array_equal(host(c), c0) and np.array_equal(host(s), s0)
        if ts0 is not None:
            assert np.array_equal(host(ts), ts0)
    # the debug and production instantiations produce the same bytes
    cd, sd, tsd, _ = W.wush_quant_act_debug(x, T, G, fmt)
    assert np.array_equal(host(cd), c0) and np.array_equal(host(sd), s0)
    y_ref = O.block_transform(O.bf16_to_f64(inp.x_bits), b["T_wush32"].astype(np.float64))
    assert_end_to_end(c0, s0, None if ts0 is None else float(ts0[0]), y_ref, fmt, G)


@pytest.mark.parametrize("name,over,fmt,G", CASES, ids=IDS)
def test_weight_bit_exact_and_end_to_end(name, over, fmt, G):
    wl, inp, b = case_data(name, over)
    w = dev_f32(inp.w)
    T = dev_f32(b["T_xvsh32"])
    c, s, ts, y = W.wush_quant_weight_debug(w, T, G, fmt)
    torch.cuda.synchronize()
    assert_device_clean()
    assert_bit_exact(host(c), host(s), ts_value(ts), host(y), fmt, G)
    c2, s2, ts2 = W.wush_quant_weight(w, T, G, fmt)
    assert np.array_equal(host(c2), host(c)) and np.array_equal(host(s2), host(s))
    y_ref = O.block_transform(inp.w.astype(np.float64), b["T_xvsh32"].astype(np.float64))
    assert_within_split_bound(host(y), y_ref, inp.w.astype(np.float64), b["T_xvsh32"], 2.0 ** -14)
    assert_end_to_end(host(c), host(s), ts_value(ts), y_ref, fmt, G)


@pytest.mark.parametrize("n_tok", [1, 17, 127, 128, 129, 255, 513])
@pytest.mark.parametrize("d_in", [32, 96, 128, 160, 4096 + 32])
def test_ragged_shapes_mxfp4(n_tok, d_in):
    wl = workload("attn_mxfp4_4096", n_tok=n_tok, d_in=d_in, d_out=64, n_cal=256,
                  n_outliers=min(2, d_in // 32))
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 32)
    c, s, ts, y = W.wush_quant_act_debug(dev_bf16(inp.x_bits), dev_f32(b["T_wush32"]), 32, "mxfp4")
    torch.cuda.synchronize()
    assert_device_clean()
    assert c.shape == (n_tok, d_in // 2) and s.shape == (n_tok, d_in // 32)
    assert_bit_exact(host(c), host(s), None, host(y), "mxfp4", 32)


@pytest.mark.parametrize("fmt,G", [("nvfp4", 16), ("int4", 16), ("int4", 32)])
@pytest.mark.parametrize("n_tok", [1, 129])
@pytest.mark.parametrize("d_in", [G_ for G_ in (32, 224)])
def test_ragged_shapes_other_formats(fmt, G, n_tok, d_in):
    wl = workload("int4_sweep_4096", n_tok=n_tok, d_in=d_in, G=G, d_out=64, n_cal=256)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, G)
    c, s, ts, y = W.wush_quant_act_debug(dev_bf16(inp.x_bits), dev_f32(b["T_wush32"]), G, fmt)
    cw, sw, tsw, yw = W.wush_quant_weight_debug(dev_f32(inp.w), dev_f32(b["T_xvsh32"]), G, fmt)
    torch.cuda.synchronize()
    assert_device_clean()
    assert_bit_exact(host(c), host(s), ts_value(ts), host(y), fmt, G)
    assert_bit_exact(host(cw), host(sw), ts_value(tsw), host(yw), fmt, G)


def test_identity_transform_quantises_input_exactly():
    """With every T_i = I the kernel's y equals x bit for bit (bf16 * 1 in fp32, lo = 0)."""
    wl = workload("attn_mxfp4_4096", n_tok=200, d_in=256, d_out=64, n_cal=64)
    inp = make_inputs(wl)
    T = np.stack([np.eye(32, dtype=np.float32)] * 8)
    c, s, ts, y = W.wush_quant_act_debug(dev_bf16(inp.x_bits), dev_f32(T), 32, "mxfp4")
    torch.cuda.synchronize()
    x = O.bf16_to_f64(inp.x_bits)
    assert np.array_equal(host(y).astype(np.float64), x)
    c_o, s_o, _ = O.quantize(x, "mxfp4", 32)
    assert np.array_equal(canon_codes(host(c), "mxfp4", packed=True), canon_codes(c_o, "mxfp4"))
    assert np.array_equal(host(s), s_o)


def test_zero_input_and_degenerate_groups():
    n, d = 130, 160
    x = np.zeros((n, d), dtype=np.uint16)
    T = np.stack([np.eye(32, dtype=np.float32)] * (d // 32))
    for fmt in ("mxfp4", "int4"):
        c, s, ts = W.wush_quant_act(dev_bf16(x), dev_f32(T), 32, fmt)
        torch.cuda.synchronize()
        assert np.all(canon_codes(host(c), fmt, packed=True) == 0)
        assert np.all(host(s) == 0)
    T16 = np.stack([np.eye(16, dtype=np.float32)] * (d // 16))
    c, s, ts = W.wush_quant_act(dev_bf16(x), dev_f32(T16), 16, "nvfp4")
    torch.cuda.synchronize()
    assert ts_value(ts) == 0.0 and np.all(host(s) == 0) and np.all(canon_codes(host(c), "nvfp4", packed=True) == 0)
    assert_device_clean()


def test_empty_batch_launches_nothing():
    T = dev_f32(np.stack([np.eye(32, dtype=np.float32)] * 4))
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    c, s, ts = W.wush_quant_act(x, T, 32, "mxfp4")
    assert c.shape == (0, 64) and s.shape == (0, 4)


def test_bounded_wait_gives_up_and_reports():
    st, bits = W.wush_selftest_wait_timeout(2_000_000)     # 2 ms
    assert st == 5 and bits == 32
    assert_device_clean()
    # the context is still usable afterwards
    T = dev_f32(np.stack([np.eye(32, dtype=np.float32)] * 4))
    x = torch.ones((5, 128), dtype=torch.bfloat16, device="cuda")
    c, s, _ = W.wush_quant_act(x, T, 32, "mxfp4")
    torch.cuda.synchronize()
    # amax 1 -> e = -2 (1 <= 6/4, 1 > 6/8): byte 125; v = 4 -> code 6 in both nibbles
    assert np.all(host(s) == 125) and np.all(host(c) == 0x66)


def test_stream_ordering_on_side_stream():
    wl, inp, b = case_data(*CASES[1][:2])
    x = dev_bf16(inp.x_bits)
    T = dev_f32(b["T_wush32"])
    ref = [host(t) for t in W.wush_quant_act(x, T, 32, "mxfp4")[:2]]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        c, sc, _ = W.wush_quant_act(x, T, 32, "mxfp4")
    s.synchronize()
    assert np.array_equal(host(c), ref[0]) and np.array_equal(host(sc), ref[1])


def test_runs_across_several_column_tiles():
    """128 rows by 57,344 channels: 448 tiles of one row tile each, so every CTA's run
    crosses three or four column tiles and refills both transform slots (a slot's second
    and later fills wait on barrier phases its first fill left behind)."""
    n, d, G = 128, 57344, 32
    g = np.random.default_rng(31)
    x = dev_bf16(bf16_bits_from_f64(g.standard_normal((n, d))))
    T = torch.from_numpy((np.eye(G, dtype=np.float32)[None] +
                          0.05 * g.standard_normal((d // G, G, G)).astype(np.float32))).cuda()
    c, s, _, y = W.wush_quant_act_debug(x, T, G, "mxfp4")
    torch.cuda.synchronize()
    assert_device_clean()
    assert_bit_exact(host(c), host(s), None, host(y).astype(np.float64), "mxfp4", G)
