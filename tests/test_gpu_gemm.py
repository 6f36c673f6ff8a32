"""MXFP4 / NVFP4 GEMM consumers and the scale-atom relayout vs the fp64 oracle (needs a B200).

D = deq(A) deq(B)^T (paper-graph-ui analysis, section 3.4.7 "GPU Kernel Design": the
FP4 MatMul that follows WUSH + Quant).  The kernel accumulates in fp32 and rounds D once
to bf16, so each element must lie within 2^-8 |D| (bf16 rounding) plus the fp32
accumulation bound K 2^-23 (|A| |B|^T) of the oracle's value (NVFP4: K + 2, for the
product of the tensor scales and the product with it).
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def random_operand(rows, K, seed, lo=120, hi=134):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.integers(lo, hi, (rows, K // 32), dtype=np.uint8)
    return codes, scales


def assert_gemm_close(d_gpu, a_c, a_s, b_c, b_s, K):
    ref = O.gemm_mx(a_c, a_s, b_c, b_s)
    A = np.abs(O.dequant(O.unpack_nibbles(a_c), a_s, "mxfp4", 32))
    B = np.abs(O.dequant(O.unpack_nibbles(b_c), b_s, "mxfp4", 32))
    bound = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -23 * (A @ B.T) + 1e-30
    err = np.abs(d_gpu.astype(np.float64) - ref)
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), f"at {worst}: gpu {d_gpu[worst]} oracle {ref[worst]} bound {bound[worst]}"


@pytest.mark.parametrize("rows,C", [(128, 8), (300, 10), (1024, 128)])
def test_scale_atoms_match_the_layout(rows, C):
    s = np.random.default_rng(rows).integers(0, 255, (rows, C), dtype=np.uint8)
    at = W.wush_mx_scales_to_atoms(dev(s))
    torch.cuda.synchronize()
    assert np.array_equal(at.cpu().numpy(), O.scale_atoms(s))


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 1024), (384, 768, 768), (128, 256, 4096)])
def test_gemm_random_operands(M, N, K):
    a_c, a_s = random_operand(M, K, 1)
    b_c, b_s = random_operand(N, K, 2)
    d = W.wush_gemm_mxfp4(dev(a_c), W.wush_mx_scales_to_atoms(dev(a_s)), dev(b_c), W.wush_mx_scales_to_atoms(dev(b_s)))
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    assert_gemm_close(d.float().cpu().numpy(), a_c, a_s, b_c, b_s, K)


def test_gemm_after_wush_quantisation():
    """The layer: activations and weights quantised with the WUSH transforms by the
    library's kernels, then the FP4 GEMM; the oracle multiplies the kernels' own codes."""
    wl = workload("attn_mxfp4_4096", n_tok=256, d_in=1024, d_out=512, n_cal=1024)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 32)
    x = dev(inp.x_bits.view(np.int16)).view(torch.bfloat16)
    cx, sx, _ = W.wush_quant_act(x, dev(b["T_wush32"]), 32, "mxfp4")
    cw, sw, _ = W.wush_quant_weight(dev(inp.w), dev(b["T_xvsh32"]), 32, "mxfp4")
    d = W.wush_gemm_mxfp4(cx, W.wush_mx_scales_to_atoms(sx), cw, W.wush_mx_scales_to_atoms(sw))
    torch.cuda.synchronize()
    assert_gemm_close(d.float().cpu().numpy(), cx.cpu().numpy(), sx.cpu().numpy(), cw.cpu().numpy(),
                      sw.cpu().numpy(), wl.d_in)
    # and the quantised layer approximates the full-precision one
    ref = O.bf16_to_f64(inp.x_bits) @ inp.w.astype(np.float64).T
    rel = np.linalg.norm(d.float().cpu().numpy() - ref) / np.linalg.norm(ref)
    assert rel < 0.25, rel


def test_gemm_rejects_unsupported_shapes():
    a = torch.zeros((100, 128), dtype=torch.uint8, device="cuda")
    b = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(W.WushError):
        W.wush_gemm_mxfp4(a, torch.zeros(W.atom_bytes(100, 8), dtype=torch.uint8, device="cuda"), b,
                          torch.zeros(W.atom_bytes(256, 8), dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("n_tok,d_in", [(256, 1024), (300, 416), (129, 4096 + 128)])
def test_quantiser_writes_scale_atoms_directly(n_tok, d_in):
    wl = workload("attn_mxfp4_4096", n_tok=n_tok, d_in=d_in, d_out=256, n_cal=512)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 32)
    x = dev(inp.x_bits.view(np.int16)).view(torch.bfloat16)
    T = dev(b["T_wush32"])
    c, s, _ = W.wush_quant_act(x, T, 32, "mxfp4")
    ca, at = W.wush_quant_act_mx_atoms(x, T)
    cw, sw, _ = W.wush_quant_weight(dev(inp.w), dev(b["T_xvsh32"]), 32, "mxfp4")
    cwa, atw = W.wush_quant_weight_mx_atoms(dev(inp.w), dev(b["T_xvsh32"]))
    H = W.wush_hadamard(32)
    ch, sh, _ = W.wush_quant_act_shared(x, H, 32, "mxfp4")
    cha, ath = W.wush_quant_act_shared_mx_atoms(x, H)
    torch.cuda.synchronize()
    assert torch.equal(c, ca) and torch.equal(cw, cwa) and torch.equal(ch, cha)
    # atom buffers start zeroed, so their padding matches the oracle's zero padding
    assert np.array_equal(at.cpu().numpy(), O.scale_atoms(s.cpu().numpy()))
    assert np.array_equal(atw.cpu().numpy(), O.scale_atoms(sw.cpu().numpy()))
    assert np.array_equal(ath.cpu().numpy(), O.scale_atoms(sh.cpu().numpy()))


def random_nv_operand(rows, K, seed):
    """Random E2M1 codes and E4M3 scales over the normal and subnormal range (0x01..0x7E,
    never the NaN code)."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.integers(0x01, 0x7F, (rows, K // 16), dtype=np.uint8)
    return codes, scales


def assert_gemm_nv_close(d_gpu, a_c, a_s, a_t, b_c, b_s, b_t, K):
    ref = O.gemm_nv(a_c, a_s, a_t, b_c, b_s, b_t)
    A = np.abs(O.dequant(O.unpack_nibbles(a_c), a_s, "nvfp4", 16, a_t))
    B = np.abs(O.dequant(O.unpack_nibbles(b_c), b_s, "nvfp4", 16, b_t))
    bound = 2.0 ** -8 * np.abs(ref) + (K + 2) * 2.0 ** -23 * (A @ B.T) + 1e-30
    err = np.abs(d_gpu.astype(np.float64) - ref)
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), f"at {worst}: gpu {d_gpu[worst]} oracle {ref[worst]} bound {bound[worst]}"


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 1024), (384, 768, 768), (128, 256, 4096)])
def test_gemm_nvfp4_random_operands(M, N, K):
    a_c, a_s = random_nv_operand(M, K, 3)
    b_c, b_s = random_nv_operand(N, K, 4)
    a_t, b_t = float(np.float32(0.37)), float(np.float32(1.9))
    ta = torch.tensor([a_t], dtype=torch.float32, device="cuda")
    tb = torch.tensor([b_t], dtype=torch.float32, device="cuda")
    d = W.wush_gemm_nvfp4(dev(a_c), W.wush_mx_scales_to_atoms(dev(a_s)), ta, dev(b_c),
                          W.wush_mx_scales_to_atoms(dev(b_s)), tb)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    assert_gemm_nv_close(d.float().cpu().numpy(), a_c, a_s, a_t, b_c, b_s, b_t, K)


def test_gemm_nvfp4_rejects_missing_tensor_scale_and_bad_shapes():
    a = torch.zeros((128, 128), dtype=torch.uint8, device="cuda")
    b = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    ts = torch.ones(1, dtype=torch.float32, device="cuda")
    lib = W.load_library()
    at = torch.zeros(W.atom_bytes(256, 16), dtype=torch.uint8, device="cuda")
    d = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
    st = lib.wush_gemm_nvfp4(a.data_ptr(), at.data_ptr(), None, b.data_ptr(), at.data_ptr(), ts.data_ptr(),
                             128, 256, 256, d.data_ptr(), None)
    assert st == 1
    a_bad = torch.zeros((100, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(W.WushError):
        W.wush_gemm_nvfp4(a_bad, at, ts, b, at, ts)


@pytest.mark.parametrize("n_tok,d_in", [(256, 1024), (300, 416), (129, 4096 + 64)])
def test_nvfp4_quantiser_writes_scale_atoms_directly(n_tok, d_in):
    wl = workload("attn_mxfp4_4096", n_tok=n_tok, d_in=d_in, d_out=256, n_cal=512)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 16)
    x = dev(inp.x_bits.view(np.int16)).view(torch.bfloat16)
    T = dev(b["T_wush32"])
    c, s, ts = W.wush_quant_act(x, T, 16, "nvfp4")
    ca, at, tsa = W.wush_quant_act_nv_atoms(x, T)
    cw, sw, tw = W.wush_quant_weight(dev(inp.w), dev(b["T_xvsh32"]), 16, "nvfp4")
    cwa, atw, twa = W.wush_quant_weight_nv_atoms(dev(inp.w), dev(b["T_xvsh32"]))
    torch.cuda.synchronize()
    assert torch.equal(c, ca) and torch.equal(cw, cwa)
    assert torch.equal(ts, tsa) and torch.equal(tw, twa)
    assert np.array_equal(at.cpu().numpy(), O.scale_atoms(s.cpu().numpy()))
    assert np.array_equal(atw.cpu().numpy(), O.scale_atoms(sw.cpu().numpy()))


def test_nvfp4_layer_after_wush_quantisation():
    """The NVFP4 layer end to end: both operands quantised by the library with the G = 16
    WUSH transforms straight into scale atoms, then the NVFP4 GEMM; the oracle multiplies
    the kernels' own codes, scales and tensor scales."""
    wl = workload("attn_mxfp4_4096", n_tok=256, d_in=1024, d_out=512, n_cal=1024)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 16)
    x = dev(inp.x_bits.view(np.int16)).view(torch.bfloat16)
    cx, sx, tx = W.wush_quant_act(x, dev(b["T_wush32"]), 16, "nvfp4")
    cw, sw, tw = W.wush_quant_weight(dev(inp.w), dev(b["T_xvsh32"]), 16, "nvfp4")
    _, ax, _ = W.wush_quant_act_nv_atoms(x, dev(b["T_wush32"]))
    _, aw, _ = W.wush_quant_weight_nv_atoms(dev(inp.w), dev(b["T_xvsh32"]))
    d = W.wush_gemm_nvfp4(cx, ax, tx, cw, aw, tw)
    torch.cuda.synchronize()
    assert_gemm_nv_close(d.float().cpu().numpy(), cx.cpu().numpy(), sx.cpu().numpy(), float(tx.item()),
                         cw.cpu().numpy(), sw.cpu().numpy(), float(tw.item()), wl.d_in)
    ref = O.bf16_to_f64(inp.x_bits) @ inp.w.astype(np.float64).T
    rel = np.linalg.norm(d.float().cpu().numpy() - ref) / np.linalg.norm(ref)
    assert rel < 0.25, rel


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_gemm_at_the_benchmarked_shape(fmt):
    """M = 1024, N = K = 4096 (the bench row), operands from the library's quantisers in
    the scale-atom layout; 4096 sampled outputs against the oracle's product of the same
    codes and scales (row-major scales from the row-major quantiser, which writes the same
    codes)."""
    M, N, K = 1024, 4096, 4096
    g = torch.Generator().manual_seed(11)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(N, K, generator=g) / K ** 0.5).cuda()
    G = 32 if fmt == "mxfp4" else 16
    T = (torch.eye(G) + 0.1 * torch.randn(K // G, G, G, generator=g)).cuda()
    if fmt == "mxfp4":
        cx, ax = W.wush_quant_act_mx_atoms(x, T)
        cw, aw = W.wush_quant_weight_mx_atoms(w, T)
        d = W.wush_gemm_mxfp4(cx, ax, cw, aw)
        _, sx, _ = W.wush_quant_act(x, T, G, fmt)
        _, sw, _ = W.wush_quant_weight(w, T, G, fmt)
        ts_x = ts_w = None
    else:
        cx, ax, tx = W.wush_quant_act_nv_atoms(x, T)
        cw, aw, tw = W.wush_quant_weight_nv_atoms(w, T)
        d = W.wush_gemm_nvfp4(cx, ax, tx, cw, aw, tw)
        _, sx, _ = W.wush_quant_act(x, T, G, fmt)
        _, sw, _ = W.wush_quant_weight(w, T, G, fmt)
        ts_x, ts_w = float(tx.item()), float(tw.item())
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    A = O.dequant(O.unpack_nibbles(cx.cpu().numpy()), sx.cpu().numpy(), fmt, G, ts_x)
    B = O.dequant(O.unpack_nibbles(cw.cpu().numpy()), sw.cpu().numpy(), fmt, G, ts_w)
    rng = np.random.default_rng(5)
    mi, ni = rng.integers(0, M, 4096), rng.integers(0, N, 4096)
    ref = np.einsum("ik,ik->i", A[mi], B[ni])
    mag = np.einsum("ik,ik->i", np.abs(A[mi]), np.abs(B[ni]))
    got = d.float().cpu().numpy()[mi, ni].astype(np.float64)
    bound = 2.0 ** -8 * np.abs(ref) + (K + 2) * 2.0 ** -23 * mag + 1e-30
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / bound)


@pytest.mark.parametrize("nv", [False, True])
@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (512, 768, 1024), (1024, 512, 4096)])
def test_cta_pair_kernel_equals_the_oracle_and_the_single_cta_kernel(M, N, K, nv):
    """The opt-in CTA-pair GEMM (M % 256 == 0): within the oracle bound, and equal to the
    single-CTA kernel up to fp32 accumulation order (both checked against the bound)."""
    if nv:
        a_c, a_s = random_nv_operand(M, K, 5)
        b_c, b_s = random_nv_operand(N, K, 6)
        ta = torch.tensor([0.5], dtype=torch.float32, device="cuda")
        tb = torch.tensor([1.25], dtype=torch.float32, device="cuda")
        run = lambda: W.wush_gemm_nvfp4(dev(a_c), W.wush_mx_scales_to_atoms(dev(a_s)), ta, dev(b_c),
                                        W.wush_mx_scales_to_atoms(dev(b_s)), tb)
    else:
        a_c, a_s = random_operand(M, K, 5)
        b_c, b_s = random_operand(N, K, 6)
        run = lambda: W.wush_gemm_mxfp4(dev(a_c), W.wush_mx_scales_to_atoms(dev(a_s)), dev(b_c),
                                        W.wush_mx_scales_to_atoms(dev(b_s)))
    try:
        W.wush_set_gemm_cta_pairs(True)
        d_pair = run()
        W.wush_set_gemm_cta_pairs(False)
        d_single = run()
        torch.cuda.synchronize()
    finally:
        W.wush_set_gemm_cta_pairs(False)
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    for d in (d_pair, d_single):
        if nv:
            assert_gemm_nv_close(d.float().cpu().numpy(), a_c, a_s, 0.5, b_c, b_s, 1.25, K)
        else:
            assert_gemm_close(d.float().cpu().numpy(), a_c, a_s, b_c, b_s, K)


@pytest.mark.parametrize("nv", [False, True])
def test_persistent_ctas_running_several_tiles(nv):
    """2048 x 5120 x 512: 320 output tiles on at most 148 CTAs, so each CTA runs two or
    three tiles and every ring (operand stages, TMEM scale slots, the accumulator and the
    output staging buffer) wraps across tiles; every element within the oracle bound."""
    M, N, K = 2048, 5120, 512
    if nv:
        a_c, a_s = random_nv_operand(M, K, 7)
        b_c, b_s = random_nv_operand(N, K, 8)
        a_t, b_t = float(np.float32(0.61)), float(np.float32(1.3))
        ta = torch.tensor([a_t], dtype=torch.float32, device="cuda")
        tb = torch.tensor([b_t], dtype=torch.float32, device="cuda")
        d = W.wush_gemm_nvfp4(dev(a_c), W.wush_mx_scales_to_atoms(dev(a_s)), ta, dev(b_c),
                              W.wush_mx_scales_to_atoms(dev(b_s)), tb)
    else:
        a_c, a_s = random_operand(M, K, 7)
        b_c, b_s = random_operand(N, K, 8)
        d = W.wush_gemm_mxfp4(dev(a_c), W.wush_mx_scales_to_atoms(dev(a_s)), dev(b_c),
                              W.wush_mx_scales_to_atoms(dev(b_s)))
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    if nv:
        assert_gemm_nv_close(d.float().cpu().numpy(), a_c, a_s, a_t, b_c, b_s, b_t, K)
    else:
        assert_gemm_close(d.float().cpu().numpy(), a_c, a_s, b_c, b_s, K)
