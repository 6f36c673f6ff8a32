"""Full-size parity: the production entry points at the workloads' full sizes, in the
launch configuration the benchmark times (same instantiation and grid rule: one
persistent CTA per SM, or for long bf16 MXFP4 runs the aligned grid of fewer CTAs),
against the fp64 oracle.

The oracle cannot quantise a 16384 x 8192 matrix in seconds, so these tests compare
sampled (row, block) groups that it computes one by one, and check properties that hold
at any size:
  * the debug instantiation (which also writes its fp32 y) produces the same bytes as the
    production one, so rule 1 on its y speaks for the production output;
  * rule 1 on sampled groups: oracle quantiser on the kernel's own y == kernel codes and
    scales, bit for bit (NVFP4: with the tensor scale the oracle derives from the
    kernel's own max |y| over the whole tensor, itself compared bit for bit);
  * rule 2 on sampled groups: kernel output vs the oracle's float64 transform of the
    same inputs (NVFP4: the oracle's tensor scale from its full float64 transform).
The INT4 token sweep is small enough to be compared in full.
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
from workloads.synthetic import INT4_SWEEP_TOKENS
import blockwise_adaptive_transforms_b200 as W
from parity_rules import assert_bit_exact, assert_end_to_end

pytestmark = pytest.mark.gpu

N_SAMPLES = 6000

_CACHE = {}


def case(name):
    if name not in _CACHE:
        wl = workload(name)
        inp = make_inputs(wl)
        b = O.build_transforms(inp.w, inp.xcal_bits, wl.G)
        _CACHE[name] = (wl, inp, b)
    return _CACHE[name]


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def sample_groups(n_rows, C, seed):
    """Random (row, block) pairs plus every block of the first and last rows and the
    last block of a spread of rows (tile edges, the final tile)."""
    rng = np.random.default_rng(seed)
    r = rng.integers(0, n_rows, N_SAMPLES)
    c = rng.integers(0, C, N_SAMPLES)
    edge_rows = np.array([0, n_rows - 1])
    r = np.concatenate([r, np.repeat(edge_rows, C), np.arange(0, n_rows, max(1, n_rows // 256))])
    c = np.concatenate([c, np.tile(np.arange(C), 2), np.full(len(range(0, n_rows, max(1, n_rows // 256))), C - 1)])
    return r, c


def gather(t, rows, blocks, width):
    """t viewed as [n][C][width]: the selected groups, on the host."""
    n = t.shape[0]
    v = t.reshape(n, -1, width)
    ri = torch.from_numpy(rows).cuda()
    bi = torch.from_numpy(blocks).cuda()
    return v[ri, bi].cpu().numpy()


def check_full_size(fmt, G, x_dev, T32, x_groups64, rows, blocks, quant, quant_debug, y_ref_full_amax):
    """Production vs debug bytes, then rules 1 and 2 on the sampled groups."""
    c, s, ts = quant(x_dev, dev_f32(T32), G, fmt)
    cd, sd, tsd, y = quant_debug(x_dev, dev_f32(T32), G, fmt)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    assert torch.equal(c, cd) and torch.equal(s, sd)
    if ts is not None:
        assert torch.equal(ts, tsd)
    ts_v = None if ts is None else float(ts.cpu().numpy()[0])

    c_s = gather(c, rows, blocks, G // 2)                      # [k][G/2]
    s_s = gather(s.reshape(s.shape[0], -1, 1), rows, blocks, 1)  # [k][1]
    y_s = gather(y, rows, blocks, G)                            # [k][G]

    # rule 1 on the sample (NVFP4: tensor scale from the kernel's own y, whole tensor)
    s_t1 = None
    if fmt == "nvfp4":
        s_t1 = O.nvfp4_tensor_scale(float(np.max(np.abs(y.cpu().numpy()))))
        assert np.float32(ts_v) == np.float32(s_t1), (ts_v, s_t1)
    assert_bit_exact(c_s, s_s, ts_v, y_s, fmt, G, s_t=s_t1)

    # rule 2 on the sample
    y_ref = O.transform_groups(x_groups64, T32, blocks)
    s_t2 = O.nvfp4_tensor_scale(y_ref_full_amax) if fmt == "nvfp4" else None
    assert_end_to_end(c_s, s_s, ts_v, y_ref, fmt, G, s_t_ref=s_t2)


def O_T64(T32):
    return np.asarray(T32, dtype=np.float64)


@pytest.mark.parametrize("name", ["attn_mxfp4_4096", "mlp_down_nvfp4_14336", "large_mxfp4_8192"])
def test_full_size_activations(name):
    wl, inp, b = case(name)
    n, d, G = wl.n_tok, wl.d_in, wl.G
    C = d // G
    rows, blocks = sample_groups(n, C, seed=wl.seed + 100)
    x64_groups = O.bf16_to_f64(inp.x_bits.reshape(n, C, G)[rows, blocks])
    amax_ref = 0.0
    if wl.fmt == "nvfp4":      # the oracle's tensor scale needs its full float64 transform
        amax_ref = float(np.max(np.abs(O.block_transform(O.bf16_to_f64(inp.x_bits), O_T64(b["T_wush32"])))))
    check_full_size(wl.fmt, G, dev_bf16(inp.x_bits), b["T_wush32"], x64_groups, rows, blocks,
                    W.wush_quant_act, W.wush_quant_act_debug, amax_ref)


def test_full_size_weights_8192():
    wl, inp, b = case("large_mxfp4_8192")
    d_out, d, G = inp.w.shape[0], wl.d_in, wl.G
    C = d // G
    rows, blocks = sample_groups(d_out, C, seed=wl.seed + 200)
    w_groups = inp.w.reshape(d_out, C, G)[rows, blocks].astype(np.float64)
    check_full_size(wl.fmt, G, dev_f32(inp.w), b["T_xvsh32"], w_groups, rows, blocks,
                    W.wush_quant_weight, W.wush_quant_weight_debug, 0.0)


@pytest.mark.parametrize("n_tok", INT4_SWEEP_TOKENS)
def test_int4_token_sweep_in_full(n_tok):
    wl, inp, b = case("int4_sweep_4096")
    x_bits = inp.x_bits[:n_tok]
    x = dev_bf16(x_bits)
    T = dev_f32(b["T_wush32"])
    c, s, _ = W.wush_quant_act(x, T, wl.G, "int4")
    cd, sd, _, y = W.wush_quant_act_debug(x, T, wl.G, "int4")
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    assert torch.equal(c, cd) and torch.equal(s, sd)
    assert_bit_exact(c.cpu().numpy(), s.cpu().numpy(), None, y.cpu().numpy(), "int4", wl.G)
    y_ref = O.block_transform(O.bf16_to_f64(x_bits), O_T64(b["T_wush32"]))
    assert_end_to_end(c.cpu().numpy(), s.cpu().numpy(), None, y_ref, "int4", wl.G)


@pytest.mark.parametrize("rows,d_in", [(12288, 8192), (8192, 16384), (20000, 4160)])
def test_every_group_is_written_whatever_the_grid(rows, d_in):
    # 12288 x 8192: aligned grid, half a column tile per CTA; 8192 x 16384: aligned grid, a
    # whole column tile per CTA; 20000 x 4160: no aligned grid (one CTA per SM), ragged
    # last row and column tiles.  E8M0 byte 0xFF is never emitted, so a scale still 0xFF
    # after the call marks a group that no CTA wrote.
    G, C = 32, d_in // 32
    gen = torch.Generator(device="cuda").manual_seed(rows + d_in)
    x = torch.randn(rows, d_in, device="cuda", generator=gen).to(torch.bfloat16)
    T = (torch.eye(G, device="cuda").repeat(C, 1, 1)
         + 0.05 * torch.randn(C, G, G, device="cuda", generator=gen)).float()
    codes = torch.empty((rows, d_in // 2), dtype=torch.uint8, device="cuda")
    scales = torch.full((rows, C), 0xFF, dtype=torch.uint8, device="cuda")
    W.wush_quant_act(x, T, G, "mxfp4", codes=codes, scales=scales)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    unwritten = (scales == 0xFF).nonzero()
    assert unwritten.numel() == 0, f"{unwritten.shape[0]} groups unwritten, first {unwritten[:4].tolist()}"
