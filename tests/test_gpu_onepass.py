"""One-launch NVFP4 (needs a B200): decode-sized batches on CUDA cores, larger ones on the
tensor-core kernel.

The CTAs meet once through a caller's workspace to agree on the tensor scale.  Checked:
codes, scales and tensor scale equal the staged NVFP4 call on the CUDA-core path bit for
bit; rule 2 against the fp64 oracle; the workspace is zero again after every call (two
calls in a row on one workspace); a grid too large to be resident at once is refused; the
call can be captured in a CUDA graph and replayed.  Above the CUDA-core threshold the
same checks hold against the four-launch call on the tensor-core kernel, and the variant
that writes the scales in the FP4 GEMM's scale-atom layout equals the four-launch atoms
call.
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W
from parity_rules import assert_end_to_end

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _small_path_everywhere():
    W.wush_set_small_batch_rows(1 << 20)     # the reference call takes the CUDA-core path too
    yield
    W.wush_set_small_batch_rows(-1)


def _data(n_tok, d_in, seed_shift=0):
    wl = workload("mlp_down_nvfp4_14336", n_tok=n_tok, d_in=d_in, d_out=2048, n_cal=512)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 16)
    x = torch.from_numpy(np.ascontiguousarray(inp.x_bits).view(np.int16)).cuda().view(torch.bfloat16)
    return inp, b, x, torch.from_numpy(b["T_wush32"]).cuda()


@pytest.mark.parametrize("n_tok,d_in", [(1, 1024), (7, 1040), (64, 4096), (128, 14336), (300, 2048)])
def test_one_launch_equals_the_staged_call(n_tok, d_in):
    inp, b, x, T = _data(n_tok, d_in)
    ws = W.nvfp4_workspace()
    c, s, ts = W.wush_quant_act_nvfp4_onepass(x, T, ws)
    c2, s2, ts2 = W.wush_quant_act(x, T, 16, "nvfp4")
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    assert torch.equal(ts, ts2) and torch.equal(c, c2) and torch.equal(s, s2)
    assert torch.count_nonzero(ws).item() == 0, ws
    y_ref = O.block_transform(O.bf16_to_f64(inp.x_bits), b["T_wush32"].astype(np.float64))
    assert_end_to_end(c.cpu().numpy(), s.cpu().numpy(), float(ts.item()), y_ref, "nvfp4", 16)


def test_two_calls_in_a_row_on_one_workspace():
    _, _, x1, T = _data(40, 2048)
    x2 = (x1.float() * -3.0).to(torch.bfloat16)                  # a different tensor scale
    ws = W.nvfp4_workspace()
    r1 = W.wush_quant_act_nvfp4_onepass(x1, T, ws)
    r2 = W.wush_quant_act_nvfp4_onepass(x2, T, ws)
    e1 = W.wush_quant_act(x1, T, 16, "nvfp4")
    e2 = W.wush_quant_act(x2, T, 16, "nvfp4")
    torch.cuda.synchronize()
    for r, e in ((r1, e1), (r2, e2)):
        assert all(torch.equal(a, b) for a, b in zip(r, e))
    assert not torch.equal(r1[2], r2[2])
    assert torch.count_nonzero(ws).item() == 0


def test_graph_capture_and_replay():
    _, _, x, T = _data(16, 4096)
    ws = W.nvfp4_workspace()
    out = W.wush_quant_act_nvfp4_onepass(x, T, ws)            # first call outside capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        W.wush_quant_act_nvfp4_onepass(x, T, ws, codes=out[0], scales=out[1], tensor_scale=out[2], stream=s)
    out[0].zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    e = W.wush_quant_act(x, T, 16, "nvfp4")
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(out, e))
    assert torch.count_nonzero(ws).item() == 0


def test_too_large_a_grid_is_refused():
    x = torch.zeros((128 * 64, 14336), dtype=torch.bfloat16, device="cuda")
    T = torch.zeros((896, 16, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(W.WushError) as e:
        W.wush_quant_act_nvfp4_onepass(x, T, W.nvfp4_workspace())
    assert e.value.status == 2        # WUSH_ERR_UNSUPPORTED


@pytest.mark.parametrize("n_tok,d_in", [(257, 1024), (1000, 2064), (4096, 14336)])
def test_one_launch_on_the_tensor_core_kernel_equals_the_four_launch_call(n_tok, d_in):
    """Above the CUDA-core threshold the one-launch call runs the tensor-core kernel (amax
    walk forwards, meeting, quantising walk backwards): bit-identical to wush_quant_act on
    the same kernel, workspace zero afterwards, two calls in a row on one workspace."""
    W.wush_set_small_batch_rows(-1)          # default threshold: both calls on tensor cores
    inp, b, x, T = _data(n_tok, d_in)
    ws = W.nvfp4_workspace()
    for scale in (1.0, -3.0):
        xs = x if scale == 1.0 else (x.float() * scale).to(torch.bfloat16)
        c, s, ts = W.wush_quant_act_nvfp4_onepass(xs, T, ws)
        c2, s2, ts2 = W.wush_quant_act(xs, T, 16, "nvfp4")
        torch.cuda.synchronize()
        st, bits = W.wush_device_status()
        assert st == 0 and bits == 0, f"device error word {bits:#x}"
        assert torch.equal(ts, ts2) and torch.equal(c, c2) and torch.equal(s, s2)
        assert torch.count_nonzero(ws).item() == 0, ws
    if n_tok <= 1000:   # rule 2 against the float64 path (the full-size case is held by bit-equality)
        y_ref = O.block_transform(O.bf16_to_f64(inp.x_bits), b["T_wush32"].astype(np.float64))
        c, s, ts = W.wush_quant_act_nvfp4_onepass(x, T, ws)
        torch.cuda.synchronize()
        assert_end_to_end(c.cpu().numpy(), s.cpu().numpy(), float(ts.item()), y_ref, "nvfp4", 16)


def test_one_launch_tensor_core_graph_capture():
    W.wush_set_small_batch_rows(-1)
    _, _, x, T = _data(600, 4096)
    ws = W.nvfp4_workspace()
    out = W.wush_quant_act_nvfp4_onepass(x, T, ws)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        W.wush_quant_act_nvfp4_onepass(x, T, ws, codes=out[0], scales=out[1], tensor_scale=out[2], stream=s)
    out[0].zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    e = W.wush_quant_act(x, T, 16, "nvfp4")
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(out, e))
    assert torch.count_nonzero(ws).item() == 0


@pytest.mark.parametrize("n_tok,d_in,threshold", [(1024, 4096, -1), (300, 416, -1), (130, 1024, 0)])
def test_one_launch_scale_atoms_equal_the_four_launch_atoms_call(n_tok, d_in, threshold):
    """wush_quant_act_nv_atoms_onepass (always the tensor-core kernel) against
    wush_quant_act_nv_atoms on the same kernel (threshold 0 sends small batches there too):
    codes, scale atoms (padding included) and tensor scale bit-identical; workspace zero."""
    W.wush_set_small_batch_rows(threshold)
    _, _, x, T = _data(n_tok, d_in)
    ws = W.nvfp4_workspace()
    for _ in range(2):
        c, a, ts = W.wush_quant_act_nv_atoms_onepass(x, T, ws)
        c2, a2, ts2 = W.wush_quant_act_nv_atoms(x, T)
        torch.cuda.synchronize()
        st, bits = W.wush_device_status()
        assert st == 0 and bits == 0, f"device error word {bits:#x}"
        assert torch.equal(ts, ts2) and torch.equal(c, c2) and torch.equal(a, a2)
        assert torch.count_nonzero(ws).item() == 0, ws
