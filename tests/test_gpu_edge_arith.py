"""The quantisers' short cuts at the edges of their ranges, through the C ABI on the
tensor-core kernel (needs a B200).  Each case is rule 1: the oracle's quantiser fed the
kernel's own fp32 y must give the kernel's codes and scales bit for bit.

* INT4: the scale amax / 7 is a Markstein-corrected reciprocal product for amax >= 2^-122
  and the division itself below that; groups on both sides of the threshold, and groups of
  zeros.
* NVFP4 under a caller's tensor scale: one far below amax / 2688 (the block scales
  saturate at 448), one far above (every block scale rounds to 0), one whose 6 * s_t is
  below the fp32 normal range (1 / (6 s_t) overflows: the division is used), one whose
  6 * s_t overflows, and a subnormal one whose reciprocal is still a normal number.
"""
import numpy as np
import pytest
import torch

from oracle import wush_oracle as O
import blockwise_adaptive_transforms_b200 as W
from parity_rules import assert_bit_exact

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _fused_path():
    W.wush_set_small_batch_rows(0)        # the tensor-core kernel, whatever the batch
    yield
    W.wush_set_small_batch_rows(-1)


def _bf16(a):
    t = torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.cuda()


def _transforms(C, G, seed):
    g = np.random.default_rng(seed)
    T = np.eye(G, dtype=np.float32)[None] + (0.05 * g.standard_normal((C, G, G))).astype(np.float32)
    return torch.from_numpy(T).cuda()


@pytest.mark.parametrize("G", [16, 32])
def test_int4_scale_both_sides_of_the_division_threshold(G):
    n, d = 300, 32 * G
    C = d // G
    g = np.random.default_rng(11)
    x = g.standard_normal((n, d)).astype(np.float32)
    # per block: normal values, values just above and just below 2^-122 after the
    # transform, values near the bf16 normal minimum, and all-zero blocks
    mult = np.array([1.0, 2.0 ** -120, 2.0 ** -123, 2.0 ** -125, 0.0, 2.0 ** -121, 2.0 ** 20, 2.0 ** -60])
    x *= np.repeat(mult[np.arange(C) % len(mult)], G)[None, :]
    xd, T = _bf16(x), _transforms(C, G, 12)
    c, s, _, y = W.wush_quant_act_debug(xd, T, G, "int4")
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    y = y.cpu().numpy().astype(np.float64)
    amax = np.abs(y.reshape(n, C, G)).max(axis=2)
    assert (amax >= 2.0 ** -122).any() and ((amax > 0) & (amax < 2.0 ** -122)).any() and (amax == 0).any()
    assert_bit_exact(c.cpu().numpy(), s.cpu().numpy(), None, y, "int4", G)


@pytest.mark.parametrize("case", ["saturating", "vanishing", "tiny_d6", "huge_d6", "subnormal_s_t"])
def test_nvfp4_under_a_callers_tensor_scale(case):
    n, d = 300, 1024
    C = d // 16
    g = np.random.default_rng(21)
    x = (g.standard_normal((n, d)) * np.exp(g.standard_normal(d))[None, :]).astype(np.float32)
    xd, T = _bf16(x), _transforms(C, 16, 22)
    _, _, ts_own, y = W.wush_quant_act_debug(xd, T, 16, "nvfp4")     # the kernel's y
    torch.cuda.synchronize()
    s_own = float(ts_own.item())
    s_t = {"saturating": s_own / 64.0, "vanishing": s_own * 1e6, "tiny_d6": 1e-40,
           "huge_d6": 3e38, "subnormal_s_t": 1e-39}[case]
    s_t = float(np.float32(s_t))
    ts = torch.tensor([s_t], dtype=torch.float32, device="cuda")
    c, s = W.wush_quant_act_nvfp4_with_scale(xd, T, ts)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    y = y.cpu().numpy().astype(np.float64)
    assert_bit_exact(c.cpu().numpy(), s.cpu().numpy(), s_t, y, "nvfp4", 16, s_t=s_t)
    sb = s.cpu().numpy()
    if case == "saturating":
        assert (sb == 0x7E).mean() > 0.5          # most block scales at E4M3's 448
    if case in ("vanishing", "huge_d6"):
        assert (sb == 0).all()
