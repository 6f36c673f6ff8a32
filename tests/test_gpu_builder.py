"""Device-built transforms vs the oracle's (LAPACK) construction, and the invariants the
pages fix, checked on the device result itself (needs a B200)."""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
from workloads import make_inputs, workload
import blockwise_adaptive_transforms_b200 as W

pytestmark = pytest.mark.gpu


def build_both(name, lam=0.01, use_h=True, **over):
    wl = workload(name, **over)
    inp = make_inputs(wl, n_tok=1)
    w = torch.from_numpy(inp.w).cuda()
    xcal = torch.from_numpy(inp.xcal_bits.view(np.int16)).view(torch.bfloat16).cuda()
    Tw, Tx, Tw64, Tx64, s64 = W.wush_build_transforms(w, xcal, wl.G, lam=lam, use_hadamard=use_h, want_f64=True)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0, f"device error word {bits:#x}"
    ref = O.build_transforms(inp.w, inp.xcal_bits, wl.G, lam=lam, use_hadamard=use_h)
    g = {k: t.cpu().numpy() for k, t in dict(Tw=Tw, Tx=Tx, Tw64=Tw64, Tx64=Tx64, s=s64).items()}
    return wl, g, ref


def separated(s, tol=1e-5):
    """Blocks whose singular values are pairwise separated (unique SVD up to signs)."""
    gaps = -np.diff(s, axis=1) / s[:, :1]
    return np.all(gaps > tol, axis=1)


@pytest.mark.parametrize("name,over", [
    ("tiny_mxfp4", {}),
    ("attn_mxfp4_4096", {}),
    ("mlp_down_nvfp4_14336", {}),
    ("int4_sweep_4096", {}),
    ("int4_sweep_4096", {"G": 16, "d_in": 1024}),
])
def test_device_transforms_match_oracle(name, over):
    wl, g, ref = build_both(name, **over)
    assert np.allclose(g["s"], ref["s"], rtol=1e-10, atol=0)
    ok = separated(ref["s"])
    assert ok.mean() > 0.9
    for key_g, key_r in (("Tw64", "T_wush"), ("Tx64", "T_xvsh")):
        a, b = g[key_g][ok], ref[key_r][ok]
        err = np.max(np.abs(a - b), axis=(1, 2)) / np.max(np.abs(b), axis=(1, 2))
        assert err.max() < 1e-9, (key_g, err.max())
    # fp32 outputs are the fp64 results rounded once
    assert np.array_equal(g["Tw"], g["Tw64"].astype(np.float32))
    assert np.array_equal(g["Tx"], g["Tx64"].astype(np.float32))


@pytest.mark.parametrize("name", ["tiny_mxfp4", "mlp_down_nvfp4_14336"])
def test_device_transforms_invariants(name):
    wl, g, ref = build_both(name)
    G = wl.G
    H = O.sylvester_hadamard(G)
    Sw = O.damp(ref["Sw"], 0.01)
    Sx = O.damp(ref["Sx"], 0.01)
    for i in range(g["Tw64"].shape[0]):
        Tw, Tx, s = g["Tw64"][i], g["Tx64"][i], g["s"][i]
        assert np.max(np.abs(Tx.T @ Tw - np.eye(G))) < 1e-9
        HSH = H @ np.diag(s) @ H.T
        sc = np.max(np.abs(HSH))
        assert np.max(np.abs(Tw @ Sx[i] @ Tw.T - HSH)) < 1e-8 * sc
        assert np.max(np.abs(Tx @ Sw[i] @ Tx.T - HSH)) < 1e-8 * sc


def test_device_wus_ablation_matches_oracle():
    wl, g, ref = build_both("tiny_mxfp4", use_h=False)
    ok = separated(ref["s"])
    err = np.max(np.abs(g["Tw64"][ok] - ref["T_wush"][ok])) / np.max(np.abs(ref["T_wush"]))
    assert err < 1e-9


def test_rank_deficient_without_damping_is_reported():
    """lambda = 0 with fewer calibration tokens than G: the activation second moment is
    singular, a Cholesky pivot is not positive, and the device error word says so."""
    wl = workload("tiny_mxfp4", n_cal=8)
    inp = make_inputs(wl, n_tok=1)
    w = torch.from_numpy(inp.w).cuda()
    xcal = torch.from_numpy(inp.xcal_bits.view(np.int16)).view(torch.bfloat16).cuda()
    W.wush_build_transforms(w, xcal, wl.G, lam=0.0)
    st, bits = W.wush_device_status()
    assert st == 5 and bits & 64
    # with damping the same data builds fine
    W.wush_build_transforms(w, xcal, wl.G, lam=0.01)
    st, bits = W.wush_device_status()
    assert st == 0
