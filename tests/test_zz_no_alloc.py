"""The allocation-free entry point (needs a B200): wush_quant_act_nvfp4_onepass_noalloc runs
the one-launch NVFP4 kernel on the library's static scratch.  Two calls in a row (with
different tensor scales, so a scratch left dirty by the first would show in the second)
must equal the workspace entry point bit for bit; too large a batch is refused.  This
file is collected last and passes on its own as well."""
import numpy as np
import pytest
import torch

import blockwise_adaptive_transforms_b200 as W

pytestmark = pytest.mark.gpu


def _inputs(n, d, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, d, generator=g).to(torch.bfloat16).cuda()
    T = (torch.eye(16) + 0.1 * torch.randn(d // 16, 16, 16, generator=g)).to(torch.float32).cuda()
    return x, T


def test_two_calls_in_a_row_equal_the_workspace_entry_point():
    x1, T = _inputs(48, 2048, 1)
    x2 = (x1.float() * 7.5).to(torch.bfloat16)
    r1 = W.wush_quant_act_nvfp4_onepass_noalloc(x1, T)
    r2 = W.wush_quant_act_nvfp4_onepass_noalloc(x2, T)
    ws = W.nvfp4_workspace()
    e1 = W.wush_quant_act_nvfp4_onepass(x1, T, ws)
    e2 = W.wush_quant_act_nvfp4_onepass(x2, T, ws)
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    assert st == 0 and bits == 0, f"device error word {bits:#x}"
    for r, e in ((r1, e1), (r2, e2)):
        assert all(torch.equal(a, b) for a, b in zip(r, e))
    assert not torch.equal(r1[2], r2[2])


def test_too_large_a_request_is_refused():
    x = torch.zeros((128 * 64, 14336), dtype=torch.bfloat16, device="cuda")
    T = torch.zeros((896, 16, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(W.WushError) as e:
        W.wush_quant_act_nvfp4_onepass_noalloc(x, T)
    assert e.value.status == 2        # WUSH_ERR_UNSUPPORTED
