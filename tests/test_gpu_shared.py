"""H+Quant comparator (one G x G matrix for every block) vs the fp64 oracle and vs the
per-block kernel (needs a B200).

The comparator is the pages' uniform blockwise-Hadamard baseline (paper-graph-ui
analysis, section 3.4.7 "GPU Kernel Design"; section 5 "GPU Kernel Benchmarks").  Its
oracle is the per-block transform with every T_i equal to the shared matrix.
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W
from parity_rules import assert_bit_exact, assert_end_to_end

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny_mxfp4", {}, "mxfp4", 32),
    ("attn_mxfp4_4096", dict(n_tok=300, d_in=416), "mxfp4", 32),
    ("mlp_down_nvfp4_14336", dict(n_tok=300, d_in=400, n_outliers=4), "nvfp4", 16),
    ("int4_sweep_4096", dict(n_tok=300, d_in=416), "int4", 32),
    ("int4_sweep_4096", dict(n_tok=300, d_in=400, G=16), "int4", 16),
]
IDS = [f"{c[0]}-{c[2]}{c[3]}" for c in CASES]


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def shared_matrices(G):
    """The normalised Hadamard matrix and a seeded random matrix, both rounded to fp32."""
    H32 = O.sylvester_hadamard(G).astype(np.float32)
    R32 = (np.random.default_rng(G).standard_normal((G, G)) / np.sqrt(G)).astype(np.float32)
    return {"hadamard": H32, "random": R32}


def inputs(name, over):
    wl = workload(name, **over)
    return wl, make_inputs(wl, need_w=False, need_cal=False)


@pytest.mark.parametrize("which", ["hadamard", "random"])
@pytest.mark.parametrize("name,over,fmt,G", CASES, ids=IDS)
def test_shared_matrix_rules_and_per_block_equivalence(name, over, fmt, G, which):
    wl, inp = inputs(name, over)
    C = wl.d_in // G
    M32 = shared_matrices(G)[which]
    x = dev_bf16(inp.x_bits)
    M = torch.from_numpy(M32).cuda()
    c, s, ts, y = W.wush_quant_act_shared_debug(x, M, G, fmt)
    c2, s2, ts2 = W.wush_quant_act_shared(x, M, G, fmt)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    assert torch.equal(c, c2) and torch.equal(s, s2)
    ts_v = None if ts is None else float(ts.cpu().numpy()[0])
    # rule 1: the oracle quantiser on the kernel's own y
    assert_bit_exact(c.cpu().numpy(), s.cpu().numpy(), ts_v, y.cpu().numpy(), fmt, G)
    # rule 2: the oracle's float64 transform with T_i = M for every block
    Trep = np.broadcast_to(M32.astype(np.float64), (C, G, G))
    y_ref = O.block_transform(O.bf16_to_f64(inp.x_bits), Trep)
    assert_end_to_end(c.cpu().numpy(), s.cpu().numpy(), ts_v, y_ref, fmt, G)
    # the per-block kernel fed C copies of M computes the same y and bytes
    Tblk = torch.from_numpy(np.ascontiguousarray(np.broadcast_to(M32, (C, G, G)))).cuda()
    cb, sb, tsb, yb = W.wush_quant_act_debug(x, Tblk, G, fmt)
    torch.cuda.synchronize()
    assert torch.equal(yb, y) and torch.equal(cb, c) and torch.equal(sb, s)


def test_shared_matrix_shape_is_checked():
    x = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        W.wush_quant_act_shared(x, torch.zeros((2, 32, 32), device="cuda"), 32, "mxfp4")


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_device_hadamard_equals_the_oracle_matrix(G):
    """wush_hadamard writes the oracle's normalised Sylvester matrix rounded once to fp32,
    bit for bit, in every copy."""
    want = O.sylvester_hadamard(G).astype(np.float32)
    one = W.wush_hadamard(G).cpu().numpy()
    assert one.shape == (G, G) and np.array_equal(one, want)
    many = W.wush_hadamard(G, copies=5).cpu().numpy()
    assert many.shape == (5, G, G)
    for k in range(5):
        assert np.array_equal(many[k], want)
    assert W.wush_hadamard(G, copies=0).shape == (0, G, G)
