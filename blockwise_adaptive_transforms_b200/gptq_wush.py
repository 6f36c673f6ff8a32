"""GPTQ-WUSH: offline weight quantisation with the WUSH transforms built inside GPTQ's
error-feedback schedule (paper-graph-ui analysis, section 3.4.6 "GPTQ Integration
(Algorithm 1)").  The printed formulas of that section are garbled; the steps are
re-derived from its text and the WUSH construction (Eq. (8)):

  Sigma = d_batch^-1 X X^T + lam mean(diag) I,  X' = chol(Sigma)   (global, lower)
  Y = W^T X'                                          (d_out x d_in, the target)
  for the blocks in reverse order:
    Y[:, blk] = U S_Y V^T  (pairs signed so that the largest |entry| of u_k is > 0)
    S = S_Y / sqrt(d_out)
    T_X = H S^1/2 V^T X'_ii^-1                         (the block's activation transform)
    W_bar = sqrt(d_out) H S^1/2 U^T                     (its transformed weights)
    GPTQ:  W~ = GPTQ(W_bar^T, Hessian H S H^T)         (Frantar et al., 2023)
    RTN:   W~ = q(W_bar^T)
    Y -= (GPTQ ? W~ : W_bar^T) T_X X'[blk, :]           (error feedback to earlier blocks)

The result plugs into the online path: activations go through wush_quant_act with T_X,
and the quantised transformed weights W~ (codes + scales in the library's layouts) are
the B operand of wush_gemm_mxfp4 (MXFP4) or are dequantised with wush_dequant.  Offline
host pipeline in float64 torch (on the GPU when given CUDA tensors); MXFP4 and INT4.
"""
from __future__ import annotations

import math

import torch

E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def hadamard64(G: int, device) -> torch.Tensor:
    H = torch.ones((1, 1), dtype=torch.float64, device=device)
    while H.shape[0] < G:
        H = torch.cat([torch.cat([H, H], 1), torch.cat([H, -H], 1)], 0)
    return H / math.sqrt(G)


def _mx_exponent(amax: torch.Tensor) -> torch.Tensor:
    """Smallest integer e with amax <= 6 * 2^e, clamped to [-127, 127]; amax = 0 -> -127."""
    a = torch.where(amax > 0, amax, torch.ones_like(amax))
    e = torch.ceil(torch.log2(a / 6.0))
    e = torch.where(a > 6.0 * torch.exp2(e), e + 1, e)
    e = torch.where(a <= 6.0 * torch.exp2(e - 1), e - 1, e)
    e = torch.where(amax > 0, e, torch.full_like(e, -127.0))
    return e.clamp(-127, 127)


def _e2m1(v: torch.Tensor):
    """Round to the E2M1 grid, ties to even, saturating at 6: (codes, values)."""
    a = v.abs()
    mag = torch.where(a < 2.0, torch.round(2.0 * a) / 2.0,
                      torch.where(a < 4.0, torch.round(a), 2.0 * torch.round(a / 2.0))).clamp(max=6.0)
    grid = torch.tensor(E2M1_GRID, dtype=v.dtype, device=v.device)
    idx = torch.searchsorted(grid, mag)
    codes = idx.to(torch.uint8) | (torch.signbit(v).to(torch.uint8) << 3)
    return codes, torch.where(torch.signbit(v), -mag, mag)


def _f32(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.float32).to(torch.float64)


def _group_scale(Wb: torch.Tensor, fmt: str):
    """Per-row group scale fixed from the starting values: (stored scale, multiplier to the
    grid, dequantisation factor)."""
    amax = Wb.abs().amax(dim=1)
    if fmt == "mxfp4":
        e = _mx_exponent(amax)
        return (e + 127).to(torch.uint8), torch.exp2(-e), torch.exp2(e)
    if fmt == "int4":
        s = _f32(amax / 7.0)
        inv = torch.where(s > 0, _f32(1.0 / torch.where(s > 0, s, torch.ones_like(s))), torch.zeros_like(s))
        inv = torch.where(torch.isfinite(inv), inv, torch.zeros_like(inv))
        return s.to(torch.float32), inv, s
    raise ValueError("GPTQ-WUSH supports mxfp4 and int4")


def _quant_column(w: torch.Tensor, mul: torch.Tensor, deq: torch.Tensor, fmt: str):
    if fmt == "mxfp4":
        c, val = _e2m1(w * mul)
        return c, val * deq
    q = torch.round(_f32(w * mul)).clamp(-7, 7)
    return (q.to(torch.int64) & 0xF).to(torch.uint8), q * deq


def gptq_block(Wb: torch.Tensor, Hb: torch.Tensor, fmt: str, damp_frac: float = 0.01):
    """GPTQ on one block: columns quantised in order at fixed group scales, each column's
    rounding error (over the diagonal of R, Hb^-1 = R^T R) taken off the later columns
    along row j of R.  Returns (dequantised [d_out][G], codes [d_out][G], scales [d_out])."""
    W = Wb.clone()
    G = W.shape[1]
    Hd = Hb + damp_frac * torch.trace(Hb) / G * torch.eye(G, dtype=Hb.dtype, device=Hb.device)
    R = torch.linalg.cholesky(torch.linalg.inv(Hd)).T
    sc, mul, deq = _group_scale(W, fmt)
    Q = torch.empty_like(W)
    codes = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
    for j in range(G):
        codes[:, j], Q[:, j] = _quant_column(W[:, j], mul, deq, fmt)
        err = (W[:, j] - Q[:, j]) / R[j, j]
        W[:, j + 1:] -= torch.outer(err, R[j, j + 1:])
    return Q, codes, sc


def _rtn_block(Wb: torch.Tensor, fmt: str):
    sc, mul, deq = _group_scale(Wb, fmt)
    if fmt == "mxfp4":
        codes, val = _e2m1(Wb * mul[:, None])
        return val * deq[:, None], codes, sc
    q = torch.round(_f32(Wb * mul[:, None])).clamp(-7, 7)
    return q * deq[:, None], (q.to(torch.int64) & 0xF).to(torch.uint8), sc


def gptq_wush(w: torch.Tensor, xcal: torch.Tensor, G: int, fmt: str, gptq: bool = True, lam: float = 0.01,
              use_hadamard: bool = True) -> dict:
    """w: weights [d_out][d_in] (row = output channel); xcal: calibration activations
    [n][d_in] (bf16 or float).  Returns a dict with
      T_act  fp32 [C][G][G]   activation transforms for the online kernel,
      codes  u8 [d_out][d_in/2] packed quantised transformed weights (low nibble first),
      scales [d_out][C]       (u8 E8M0 for MXFP4, fp32 for INT4),
      Wq     float64 [d_out][d_in] dequantised transformed weights,
      T_act64, residual (the final target, ~0 in RTN mode)."""
    if fmt not in ("mxfp4", "int4"):
        raise ValueError("GPTQ-WUSH supports mxfp4 and int4")
    dev = w.device
    Wt = w.to(torch.float64)
    X = xcal.to(torch.float64)
    d_out, d_in = Wt.shape
    n = X.shape[0]
    if d_in % G:
        raise ValueError("d_in must be a multiple of G")
    C = d_in // G
    Sig = X.T @ X / n
    Sig += lam * torch.trace(Sig) / d_in * torch.eye(d_in, dtype=torch.float64, device=dev)
    Xp = torch.linalg.cholesky(Sig)
    Y = Wt @ Xp
    H = hadamard64(G, dev) if use_hadamard else torch.eye(G, dtype=torch.float64, device=dev)
    T_act = torch.empty((C, G, G), dtype=torch.float64, device=dev)
    Wq = torch.empty((d_out, d_in), dtype=torch.float64, device=dev)
    codes_u = torch.empty((d_out, d_in), dtype=torch.uint8, device=dev)
    scales = torch.empty((d_out, C), dtype=torch.uint8 if fmt == "mxfp4" else torch.float32, device=dev)
    for i in reversed(range(C)):
        blk = slice(i * G, (i + 1) * G)
        U, sY, Vh = torch.linalg.svd(Y[:, blk], full_matrices=False)
        V = Vh.T
        j = U.abs().argmax(dim=0)
        sign = torch.where(U[j, torch.arange(G, device=dev)] < 0, -1.0, 1.0).to(torch.float64)
        U, V = U * sign, V * sign
        s = sY / math.sqrt(d_out)
        Xii = Xp[blk, blk]
        T_x = H @ torch.diag(s.sqrt()) @ V.T @ torch.linalg.inv(Xii)
        W_bar = math.sqrt(d_out) * H @ torch.diag(s.sqrt()) @ U.T
        if gptq:
            Q, cu, sc = gptq_block(W_bar.T.contiguous(), H @ torch.diag(s) @ H.T, fmt)
            contrib = Q
        else:
            Q, cu, sc = _rtn_block(W_bar.T.contiguous(), fmt)
            contrib = W_bar.T
        Y -= contrib @ T_x @ Xp[blk, :]
        T_act[i] = T_x
        Wq[:, blk], codes_u[:, blk], scales[:, i] = Q, cu, sc
    codes = (codes_u[:, 0::2] & 0xF) | ((codes_u[:, 1::2] & 0xF) << 4)
    return {"T_act": T_act.to(torch.float32).contiguous(), "T_act64": T_act, "codes": codes.contiguous(),
            "scales": scales.contiguous(), "Wq": Wq, "residual": Y}
