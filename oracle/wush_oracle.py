"""Independent float64 CPU oracle for WUSH blockwise transforms + 4-bit quantisation.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
test-suite, the smoke check and the benchmark's CPU-baseline leg (and its
``--impl reference`` arm) may import or run it.  It shares no code with the CUDA
path: it has its own Hadamard, second moments, factorisations (numpy LAPACK
Cholesky and SVD used as plain library steps), transform, grids and quantisers.

Sources, cited as page + section (all five pages describe arXiv 2512.00956,
"WUSH: Near-Optimal Adaptive Transforms for LLM Quantization"):
  [notes]   papernotes.org summary, sections "整体框架" and "关键设计"
  [ai.info] ai.info AI summary, "Key Contributions" / "Main Findings" /
            "Methodology in Plain English"
  [gist]    gist.science explainer, "Technisches Resümee" §2 "Methodik"
  [graph]   paper-graph-ui analysis, §3.2 "Big-Picture Architecture",
            §3.4.1-§3.4.7 (problem, reduction, parameterisation, FP/INT analysis,
            GPTQ integration, GPU kernel design)

Readings where the pages are silent, garbled or at odds (each also listed in the
design notes of the repository):
  R1  Activations use T_wush = H S^-1/2 U^T W'^T and weights T_xvsh = H S^-1/2 V^T X'^T
      ([notes] 关键设计, [graph] §3.2 and §3.4.2 where T_X = T W'^T with
      T = H S^-1/2 U^T); [gist] §2 prints the labels the other way round.
  R2  Damping: Sigma <- Sigma + lam * mean(diag Sigma) * I on both sides, lam = 0.01
      by default (the pages name a damping factor, [ai.info] Methodology and
      [graph] §3.4.6, but give no value or form).
  R3  SVD sign convention: each pair (u_k, v_k) is flipped so that the entry of
      largest magnitude of u_k is positive (ties -> lowest index).
  R4  E2M1 rounding is round-to-nearest with ties to the even code, magnitude
      saturates at 6; codes 0x0 and 0x8 are both zero.
  R5  MXFP4 scale: the smallest power of two 2^e with amax <= 6 * 2^e, e clamped to
      [-127, 127], amax = 0 -> e = -127; stored as the E8M0 byte e + 127.
  R6  NVFP4: tensor scale s_t = fl32(amax_tensor / (6 * 448)); per group
      r = fl32(amax / fl32(6 s_t)), block scale byte = E4M3(r) (RNE, satfinite,
      subnormals kept); v = fl32(y * fl32(1 / fl32(dec(sb) * s_t))).
  R7  INT4: symmetric, s = fl32(amax / 7), v = fl32(y * fl32(1 / s)), q = clamp(RNE(v), -7, 7),
      stored as a two's-complement nibble with an fp32 scale.  ([graph] §3.4.5 writes
      the scale as 2^(1-b) * amax, i.e. amax / 8, which would need the code +8.)
  R8  Packing: byte j holds element 2j in its low nibble and 2j+1 in its high nibble.
  R9  A group whose scale reciprocal fl32(1/S) is not a finite float32 (S = 0, or S so
      small that 1/S overflows) encodes as all zero codes (the pages are silent).
  R12 GPTQ-WUSH: the target is Y = W^T X' with X' the Cholesky factor of the damped global
      second moment; per block (reverse order) the SVD of Y's block gives U, S_Y, V,
      S = S_Y / sqrt(d_out), T_X = H S^1/2 V^T X'_ii^-1, transformed weights
      sqrt(d_out) H S^1/2 U^T, GPTQ with the block Hessian H S H^T (damped 1 %), and
      Y -= (quantised weights)^T T_X X'[blk, :] ([graph] §3.4.6, whose formulas are
      garbled; re-derived from its text and Eq. (8)).  GPTQ-WUSH covers MXFP4 and INT4.
fl32(.) marks a float32 rounding point: the oracle computes in float64 and rounds
to float32 there, which equals the IEEE float32 result of a single +, -, *, /.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------


def fl32(a):
    """Round float64 value(s) to the nearest float32 and return them as float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode bfloat16 bit patterns (uint16) exactly to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# transform construction
# ---------------------------------------------------------------------------


def sylvester_hadamard(G: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix of order G (a power of two).

    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]], scaled by G^-1/2 so that every
    entry is +-G^-1/2 and H H^T = I ([graph] §3.4.4, the choice U' = H).
    """
    if G < 1 or G & (G - 1):
        raise ValueError("G must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < G:
        H = np.block([[H, H], [H, -H]])
    return H / np.sqrt(G)


def block_second_moments(w: np.ndarray, xcal: np.ndarray, G: int):
    """Per-block uncentred second moments.

    Sigma_w,i = d_out^-1 W_(i) W_(i)^T and Sigma_x,i = d_batch^-1 X_(i) X_(i)^T, where
    W_(i) (G x d_out) and X_(i) (G x d_batch) are the rows of block i of the
    pages' W in R^{d_in x d_out} and X in R^{d_in x d_batch} ([notes] 关键设计;
    [graph] §3.2 "Second-Moment Computer").  Here ``w`` is stored [d_out][d_in]
    (one row per output channel) and ``xcal`` [d_batch][d_in] (one row per token),
    i.e. the transposes of the pages' matrices.
    """
    w = np.asarray(w, dtype=np.float64)
    xcal = np.asarray(xcal, dtype=np.float64)
    d_out, d_in = w.shape
    n = xcal.shape[0]
    C = d_in // G
    Sw = np.empty((C, G, G))
    Sx = np.empty((C, G, G))
    for i in range(C):
        Wi = w[:, i * G:(i + 1) * G].T          # G x d_out
        Xi = xcal[:, i * G:(i + 1) * G].T       # G x d_batch
        Sw[i] = Wi @ Wi.T / d_out
        Sx[i] = Xi @ Xi.T / n
    return Sw, Sx


def damp(S: np.ndarray, lam: float) -> np.ndarray:
    """Reading R2: Sigma + lam * mean(diag Sigma) * I (per block)."""
    S = np.array(S, dtype=np.float64, copy=True)
    G = S.shape[-1]
    for i in range(S.shape[0]):
        S[i] += lam * np.trace(S[i]) / G * np.eye(G)
    return S


def transforms_from_moments(Sw: np.ndarray, Sx: np.ndarray, use_hadamard: bool = True):
    """WUSH transforms of every block from its (damped) second moments.

    Steps ([graph] §3.2 "Transform Constructor", §3.4.2 and §3.4.4 Eq. (8);
    [notes] 关键设计; [ai.info] Methodology):
      W' = chol(Sigma_w), X' = chol(Sigma_x)     lower triangular
      W'^T X' = U S V^T                            SVD, s_1 >= ... >= s_G > 0
      T_wush = H S^-1/2 U^T W'^T                   applied to activations (R1)
      T_xvsh = H S^-1/2 V^T X'^T                   applied to weights
    ``use_hadamard=False`` replaces H by I (the pages' WUS ablation).
    Returns a dict of float64 arrays: T_wush, T_xvsh [C][G][G], s [C][G], U, V, Wp, Xp.
    """
    C, G, _ = Sw.shape
    H = sylvester_hadamard(G) if use_hadamard else np.eye(G)
    out = {k: np.empty((C, G, G)) for k in ("T_wush", "T_xvsh", "U", "V", "Wp", "Xp")}
    out["s"] = np.empty((C, G))
    for i in range(C):
        Wp = np.linalg.cholesky(Sw[i])
        Xp = np.linalg.cholesky(Sx[i])
        U, s, Vt = np.linalg.svd(Wp.T @ Xp)
        V = Vt.T
        for k in range(G):                       # reading R3
            j = int(np.argmax(np.abs(U[:, k])))
            if U[j, k] < 0:
                U[:, k] = -U[:, k]
                V[:, k] = -V[:, k]
        Sm = np.diag(s ** -0.5)
        out["T_wush"][i] = H @ Sm @ U.T @ Wp.T
        out["T_xvsh"][i] = H @ Sm @ V.T @ Xp.T
        out["s"][i], out["U"][i], out["V"][i], out["Wp"][i], out["Xp"][i] = s, U, V, Wp, Xp
    return out


def build_transforms(w: np.ndarray, xcal_bits: np.ndarray, G: int, lam: float = 0.01,
                     use_hadamard: bool = True):
    """Transforms of a layer from its weights (fp32 [d_out][d_in]) and bfloat16
    calibration activations ([n_cal][d_in] bit patterns): second moments, damping,
    then ``transforms_from_moments``.  The float32 copies handed to a kernel are
    the float64 results rounded once (``out["T_wush32"]``, ``out["T_xvsh32"]``)."""
    Sw, Sx = block_second_moments(w, bf16_to_f64(xcal_bits), G)
    out = transforms_from_moments(damp(Sw, lam), damp(Sx, lam), use_hadamard)
    out["Sw"], out["Sx"] = Sw, Sx
    out["T_wush32"] = out["T_wush"].astype(np.float32)
    out["T_xvsh32"] = out["T_xvsh"].astype(np.float32)
    return out


# ---------------------------------------------------------------------------
# the online transform
# ---------------------------------------------------------------------------


def block_transform(x: np.ndarray, T: np.ndarray) -> np.ndarray:
    """y = T_i x per token and block ([graph] §3.2 "Online Activation Transform",
    §3.4.7: per token t and block i, y[t, iG + r] = sum_c T_i[r, c] x[t, iG + c]).

    ``x`` is [n][d_in] (one row per token, or per output channel for weights) and
    ``T`` is [C][G][G]; everything is evaluated in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    T = np.asarray(T, dtype=np.float64)
    C, G, _ = T.shape
    n, d = x.shape
    if d != C * G:
        raise ValueError("d_in must equal C * G")
    xr = x.reshape(n, C, G)
    y = np.einsum("crk,nck->ncr", T, xr, optimize=True)
    return y.reshape(n, d)


def transform_groups(x_groups: np.ndarray, T: np.ndarray, blocks: np.ndarray) -> np.ndarray:
    """The same y = T_i x for a list of single (token, block) groups: row k of
    ``x_groups`` ([k][G]) is the input group of block ``blocks[k]``; float64."""
    xg = np.asarray(x_groups, dtype=np.float64)
    Tb = np.asarray(T, dtype=np.float64)[np.asarray(blocks)]
    return np.einsum("krc,kc->kr", Tb, xg)


# ---------------------------------------------------------------------------
# 4-bit grids and scale encodings
# ---------------------------------------------------------------------------

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Round to the E2M1 grid (reading R4) and return 4-bit codes (bit 3 = sign).

    Round-to-nearest-even on each binade: spacing 0.5 on [0, 2), 1 on [2, 4),
    2 on [4, 6]; numpy's rint rounds half to even, which on this grid lands on the
    code with an even index; magnitudes above 6 saturate to 6.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    mag = np.where(a < 2.0, np.rint(2.0 * a) / 2.0,
                   np.where(a < 4.0, np.rint(a), 2.0 * np.rint(a / 2.0)))
    mag = np.minimum(mag, 6.0)
    idx = np.searchsorted(E2M1_GRID, mag).astype(np.uint8)
    return idx | (np.signbit(v).astype(np.uint8) << np.uint8(3))


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_GRID[c & 7]
    return np.where(c & 8, -mag, mag)


def e4m3_encode(r: np.ndarray) -> np.ndarray:
    """Round to FP8 E4M3 (bias 7, 3 mantissa bits, max 448, subnormal spacing 2^-9),
    round-to-nearest-even, saturating at 448; returns the byte."""
    r = np.asarray(r, dtype=np.float64)
    a = np.abs(r)
    _, k = np.frexp(np.where(a > 0, a, 1.0))
    E = np.maximum(k - 1, -6)                       # binade exponent; subnormals use 2^-6
    q = np.ldexp(1.0, E - 3)                        # spacing in that binade
    m = np.minimum(np.rint(a / q) * q, 448.0)
    m = np.where(a > 0, m, 0.0)
    _, km = np.frexp(np.where(m > 0, m, 1.0))
    Em = km - 1
    normal = m >= 2.0 ** -6
    exp_field = np.where(normal, Em + 7, 0)
    mant = np.where(normal, np.rint(m / np.ldexp(1.0, Em) * 8.0 - 8.0), np.rint(m / 2.0 ** -9))
    byte = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    byte = byte | (np.signbit(r).astype(np.int64) << 7)
    return byte.astype(np.uint8)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    e = (b >> 3) & 0xF
    m = b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    if np.any((b & 0x7F) == 0x7F):
        raise ValueError("E4M3 NaN encoding")
    return np.where(b & 0x80, -mag, mag)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Reading R8: [n][d] 4-bit codes -> [n][d/2] bytes, low nibble = even element."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


# ---------------------------------------------------------------------------
# AbsMax round-to-nearest block quantisers ([ai.info] abstract: "RTN AbsMax-scaled
# block quantizers"; [graph] §3.4.1 groups of d = 32 for MXFP4 and 16 for NVFP4,
# §3.4.5 AbsMax scale from the block maximum)
# ---------------------------------------------------------------------------


def _groups(y: np.ndarray, g: int) -> np.ndarray:
    y = np.asarray(y, dtype=np.float64)
    n, d = y.shape
    if d % g:
        raise ValueError("width must be a multiple of the group size")
    return y.reshape(n, d // g, g)


def mxfp4_exponent(amax: np.ndarray, rule: str = "absmax") -> np.ndarray:
    """Reading R5: e = min{e in Z : amax <= 6 * 2^e}, clamped to [-127, 127].

    ``rule="ocp_floor"`` gives the OCP MX alternative e = floor(log2 amax) - 2,
    which lets values in (6, 8) * 2^e saturate; it is kept only for comparison.
    """
    amax = np.asarray(amax, dtype=np.float64)
    pos = amax > 0
    a = np.where(pos, amax, 1.0)
    if rule == "absmax":
        e = np.ceil(np.log2(a / 6.0))
        e = np.where(a > 6.0 * np.exp2(e), e + 1, e)          # enforce the definition exactly
        e = np.where(a <= 6.0 * np.exp2(e - 1), e - 1, e)
    elif rule == "ocp_floor":
        _, k = np.frexp(a)
        e = (k - 1) - 2.0
    else:
        raise ValueError(rule)
    e = np.where(pos, e, -127.0)
    return np.clip(e, -127, 127).astype(np.int64)


def quant_mxfp4(y: np.ndarray, rule: str = "absmax"):
    """MXFP4: groups of 32, E8M0 scale byte e + 127, codes E2M1(y * 2^-e).
    Returns (codes [n][d] uint8 nibbles, scales [n][d/32] uint8)."""
    g = _groups(y, 32)
    e = mxfp4_exponent(np.max(np.abs(g), axis=2), rule)
    v = g * np.exp2(-e.astype(np.float64))[:, :, None]        # exact in float64
    codes = e2m1_encode(v).reshape(y.shape)
    return codes, (e + 127).astype(np.uint8)


def _recip32(S: np.ndarray) -> np.ndarray:
    """fl32(1 / S) for S > 0; 0 where S is 0 or where the float32 reciprocal overflows
    (reading R9: such a group encodes as all zero)."""
    S = np.asarray(S, dtype=np.float64)
    with np.errstate(divide="ignore", over="ignore"):
        inv = np.where(S > 0, np.float32(1.0) / np.where(S > 0, S, 1.0).astype(np.float32), 0.0)
    inv = np.asarray(inv, dtype=np.float64)
    return np.where(np.isfinite(inv), inv, 0.0)


def nvfp4_tensor_scale(amax_tensor: float) -> float:
    """Reading R6: s_t = fl32(amax_tensor / 2688), 2688 = 6 * 448."""
    return float(fl32(np.float64(amax_tensor) / 2688.0))


def quant_nvfp4(y: np.ndarray, s_t: float | None = None):
    """NVFP4: groups of 16, E4M3 block scale under the fp32 tensor scale s_t (R6).
    Returns (codes [n][d] nibbles, scales [n][d/16] E4M3 bytes, s_t)."""
    g = _groups(y, 16)
    if s_t is None:
        s_t = nvfp4_tensor_scale(np.max(np.abs(g)) if g.size else 0.0)
    amax = np.max(np.abs(g), axis=2)
    d6 = fl32(6.0 * s_t)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(d6 > 0, fl32(amax / d6), 0.0)
    sb = e4m3_encode(r)
    S = fl32(e4m3_decode(sb) * s_t)
    inv = _recip32(S)
    v = fl32(g * inv[:, :, None])
    codes = e2m1_encode(v).reshape(y.shape)
    return codes, sb, s_t


def quant_int4(y: np.ndarray, G: int):
    """Symmetric INT4 AbsMax (R7).  Returns (codes [n][d] nibbles, scales [n][d/G] fp32)."""
    g = _groups(y, G)
    amax = np.max(np.abs(g), axis=2)
    s = fl32(amax / 7.0)
    inv = _recip32(s)
    v = fl32(g * inv[:, :, None])
    q = np.clip(np.rint(v), -7, 7).astype(np.int64)
    codes = (q & 0xF).astype(np.uint8).reshape(y.shape)
    return codes, s.astype(np.float32)


def int4_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64) & 0xF
    return np.where(c >= 8, c - 16, c).astype(np.float64)


# ---------------------------------------------------------------------------
# dequantisation and the composed path
# ---------------------------------------------------------------------------


def dequant(codes: np.ndarray, scales: np.ndarray, fmt: str, G: int, s_t: float | None = None):
    """Float64 values represented by unpacked codes and their scales."""
    n, d = codes.shape
    if fmt == "mxfp4":
        sc = np.exp2(np.asarray(scales, dtype=np.float64) - 127.0)
        return (e2m1_decode(codes).reshape(n, d // 32, 32) * sc[:, :, None]).reshape(n, d)
    if fmt == "nvfp4":
        sc = e4m3_decode(scales) * float(s_t)
        return (e2m1_decode(codes).reshape(n, d // 16, 16) * sc[:, :, None]).reshape(n, d)
    if fmt == "int4":
        sc = np.asarray(scales, dtype=np.float64)
        return (int4_decode(codes).reshape(n, d // G, G) * sc[:, :, None]).reshape(n, d)
    raise ValueError(fmt)


def quantize(y: np.ndarray, fmt: str, G: int):
    """Quantise transformed values y with the format's AbsMax rule.
    Returns (unpacked codes, scales, tensor scale or None)."""
    if fmt == "mxfp4":
        if G != 32:
            raise ValueError("MXFP4 groups are 32 wide")
        c, s = quant_mxfp4(y)
        return c, s, None
    if fmt == "nvfp4":
        if G != 16:
            raise ValueError("NVFP4 groups are 16 wide")
        return quant_nvfp4(y)
    if fmt == "int4":
        c, s = quant_int4(y, G)
        return c, s, None
    raise ValueError(fmt)


def quant_act(x_bits: np.ndarray, T32: np.ndarray, G: int, fmt: str):
    """The whole online path on one batch: bfloat16 activations -> per-block
    transform with the float32 T (evaluated in float64) -> AbsMax quantisation.
    Returns (packed codes [n][d/2], scales, tensor scale or None, y float64)."""
    y = block_transform(bf16_to_f64(x_bits), np.asarray(T32, dtype=np.float64))
    c, s, st = quantize(y, fmt, G)
    return pack_nibbles(c), s, st, y


def quant_weight(w: np.ndarray, T32: np.ndarray, G: int, fmt: str):
    """Weight pre-quantisation: W_bar = T_xvsh,i W_(i) per block, then RTN AbsMax
    ([notes] 整体框架; [graph] §3.2 "Weight Pre-Quantizer", §3.4.6 RTN branch).
    ``w`` is float32 [d_out][d_in].  Returns the same tuple as ``quant_act``."""
    y = block_transform(np.asarray(w, dtype=np.float64), np.asarray(T32, dtype=np.float64))
    c, s, st = quantize(y, fmt, G)
    return pack_nibbles(c), s, st, y


def layer_loss(w: np.ndarray, x_bits: np.ndarray, T_w32: np.ndarray, T_x32: np.ndarray,
               fmt: str, G: int) -> float:
    """Layerwise RTN quantisation loss ([graph] §3.4.1, the normalised Frobenius loss of
    Eq. (5); §5 "Metrics" and "Per-Layer Quantization Loss (Table 1)"):

        L = || W^T X - q(T_W W)^T q(T_X X) ||_F^2 / (d_out d_batch)

    with the pages' W [d_in][d_out] and X [d_in][d_batch].  Here, in row layouts,
    ``w`` is float32 [d_out][d_in] (one row per output channel), ``x_bits`` bfloat16
    [d_batch][d_in] (one row per token); T_W acts on the weight rows' blocks and T_X on
    the tokens' blocks, each rounded once to float32; q is the format's RTN AbsMax
    quantiser followed by dequantisation ("fake quantisation", [graph] §5 Metrics).
    Everything in float64."""
    w64 = np.asarray(w, dtype=np.float64)
    x64 = bf16_to_f64(x_bits)
    cw, sw, tw, _ = quant_weight(w, T_w32, G, fmt)
    cx, sx, tx, _ = quant_act(x_bits, T_x32, G, fmt)
    wq = dequant(unpack_nibbles(cw), sw, fmt, G, tw)
    xq = dequant(unpack_nibbles(cx), sx, fmt, G, tx)
    err = w64 @ x64.T - wq @ xq.T
    return float(np.sum(err * err) / err.size)


# ---------------------------------------------------------------------------
# GPTQ-WUSH (offline weight quantisation with error feedback)
# ---------------------------------------------------------------------------


def _group_scale(Wb: np.ndarray, fmt: str):
    """Per-row scale of one G-wide group, fixed from the row's starting values: MXFP4
    2^e (R5), INT4 s = fl32(amax / 7) (R7).  Returns (scale bytes or values, multiplier
    used to reach the grid, dequantisation factor)."""
    amax = np.max(np.abs(Wb), axis=1)
    if fmt == "mxfp4":
        e = mxfp4_exponent(amax)
        return (e + 127).astype(np.uint8), np.exp2(-e.astype(np.float64)), np.exp2(e.astype(np.float64))
    if fmt == "int4":
        sc = fl32(amax / 7.0)
        return sc.astype(np.float32), _recip32(sc), sc
    raise ValueError("GPTQ-WUSH supports mxfp4 and int4")


def _quant_column(w: np.ndarray, mul: np.ndarray, deq: np.ndarray, fmt: str):
    """One column of a block (one element of every row's group) at the fixed scales:
    (codes, dequantised values)."""
    if fmt == "mxfp4":
        c = e2m1_encode(w * mul)                     # exact: power-of-two multiplier
        return c, e2m1_decode(c) * deq
    v = fl32(w * mul)
    q = np.clip(np.rint(v), -7, 7)
    return (q.astype(np.int64) & 0xF).astype(np.uint8), q * deq


def gptq_block(Wb: np.ndarray, Hb: np.ndarray, fmt: str, damp_frac: float = 0.01):
    """GPTQ on one block (Frantar et al., 2023, restated): the block's columns are
    quantised one after the other at the group scales fixed from the starting values;
    the rounding error of column j, divided by the j-th diagonal of the upper Cholesky
    factor R of Hb^-1 (Hb^-1 = R^T R), is taken off the later columns in proportion to
    row j of R.  ``Wb`` is [d_out][G] (rows = output channels), ``Hb`` [G][G] is damped by
    damp_frac * mean(diag) (the usual GPTQ damping).
    Returns (dequantised [d_out][G], unpacked codes [d_out][G], scales [d_out])."""
    W = np.array(Wb, dtype=np.float64, copy=True)
    G = W.shape[1]
    Hd = np.asarray(Hb, dtype=np.float64) + damp_frac * np.trace(Hb) / G * np.eye(G)
    R = np.linalg.cholesky(np.linalg.inv(Hd)).T
    sc, mul, deq = _group_scale(W, fmt)
    Q = np.empty_like(W)
    codes = np.empty(W.shape, np.uint8)
    for j in range(G):
        codes[:, j], Q[:, j] = _quant_column(W[:, j], mul, deq, fmt)
        err = (W[:, j] - Q[:, j]) / R[j, j]
        W[:, j + 1:] -= np.outer(err, R[j, j + 1:])
    return Q, codes, sc


def gptq_wush(w: np.ndarray, xcal_bits: np.ndarray, G: int, fmt: str, gptq: bool = True, lam: float = 0.01,
              use_hadamard: bool = True):
    """GPTQ-WUSH, the pages' interleaved schedule ([graph] §3.4.6 "GPTQ Integration
    (Algorithm 1)"; the printed formulas are garbled, the steps below are re-derived from
    the surrounding text and Eq. (8), reading R12):

      Sigma = d_batch^-1 X X^T + lam mean(diag) I,  X' = chol(Sigma) (global, lower),
      Y = W^T X'                                   (d_out x d_in, the target)
      for blocks i = C-1 .. 0 (reverse):
        Y[:, blk] = U S_Y V^T,  S = S_Y / sqrt(d_out)   (sign rule R3 on U's columns)
        T_X = H S^1/2 V^T X'_ii^-1                  (activation transform, online)
        T_W = H S^-1/2 V^T X'_ii^T                  (T_W^T T_X = I)
        W_bar = sqrt(d_out) H S^1/2 U^T              (= T_W applied to the block's
                                                      effective weights, G x d_out)
        GPTQ: W~ = GPTQ(W_bar^T, H S H^T);  RTN: W~ = q(W_bar^T)
        Y -= (GPTQ ? W~ : W_bar^T) T_X X'[blk, :]    (error feedback to earlier blocks)

    Inputs as in ``layer_loss``: w float32 [d_out][d_in], xcal_bits bfloat16 [n][d_in].
    Returns a dict: T_act, T_w [C][G][G]; W_bar [C][G][d_out]; Wq [d_out][d_in]
    (dequantised transformed weights); codes [d_out][d_in/2] packed; scales [d_out][C];
    Y (the final residual target)."""
    Wt = np.asarray(w, dtype=np.float64)                    # [d_out][d_in] = W^T
    X = bf16_to_f64(xcal_bits)                              # [n][d_in] = X^T
    d_out, d_in = Wt.shape
    n = X.shape[0]
    C = d_in // G
    Sig = X.T @ X / n
    Sig += lam * np.trace(Sig) / d_in * np.eye(d_in)
    Xp = np.linalg.cholesky(Sig)
    Y = Wt @ Xp
    H = sylvester_hadamard(G) if use_hadamard else np.eye(G)
    out = {"T_act": np.empty((C, G, G)), "T_w": np.empty((C, G, G)), "W_bar": np.empty((C, G, d_out)),
           "Wq": np.empty((d_out, d_in)), "codes_u": np.empty((d_out, d_in), np.uint8),
           "scales": np.empty((d_out, C), np.uint8 if fmt == "mxfp4" else np.float32)}
    for i in reversed(range(C)):
        blk = slice(i * G, (i + 1) * G)
        U, sY, Vt = np.linalg.svd(Y[:, blk], full_matrices=False)
        V = Vt.T
        for k in range(G):                       # reading R3 on the columns of U
            j = int(np.argmax(np.abs(U[:, k])))
            if U[j, k] < 0:
                U[:, k] = -U[:, k]
                V[:, k] = -V[:, k]
        s = sY / np.sqrt(d_out)
        Xii = Xp[blk, blk]
        T_x = H @ np.diag(np.sqrt(s)) @ V.T @ np.linalg.inv(Xii)
        T_w = H @ np.diag(1.0 / np.sqrt(s)) @ V.T @ Xii.T
        W_bar = np.sqrt(d_out) * H @ np.diag(np.sqrt(s)) @ U.T
        if gptq:
            Q, cu, sc = gptq_block(W_bar.T, H @ np.diag(s) @ H.T, fmt)
            contrib = Q
        else:
            cu, sc = quantize(W_bar.T, fmt, G)[:2]
            Q = dequant(cu, sc.reshape(-1, 1), fmt, G)
            sc = sc.reshape(-1)
            contrib = W_bar.T
        Y -= contrib @ T_x @ Xp[blk, :]
        out["T_act"][i], out["T_w"][i], out["W_bar"][i] = T_x, T_w, W_bar
        out["Wq"][:, blk], out["codes_u"][:, blk], out["scales"][:, i] = Q, cu, sc
    out["codes"] = pack_nibbles(out.pop("codes_u"))
    out["Y"] = Y
    return out


def layer_loss_prequantised(wq: np.ndarray, w: np.ndarray, x_bits: np.ndarray, T_x32: np.ndarray,
                            fmt: str, G: int) -> float:
    """Eq. (5) when the transformed weights are already quantised (GPTQ-WUSH):
    || W^T X - Wq^T q(T_X X) ||_F^2 / (d_out d_batch), wq [d_out][d_in] dequantised."""
    x64 = bf16_to_f64(x_bits)
    cx, sx, tx, _ = quant_act(x_bits, T_x32, G, fmt)
    xq = dequant(unpack_nibbles(cx), sx, fmt, G, tx)
    err = np.asarray(w, dtype=np.float64) @ x64.T - np.asarray(wq, dtype=np.float64) @ xq.T
    return float(np.sum(err * err) / err.size)


def scale_atoms(scales: np.ndarray) -> np.ndarray:
    """One-byte scales [rows][C] (E8M0 or E4M3) in the block-scaled MMA's scale-atom
    layout (a hardware format, not from the pages): rows padded to a multiple of 128 and C to a multiple
    of 4 with zero bytes; row 128 r + i + 32 j, column 4 c + k goes to byte
    (r * C_pad / 4 + c) * 512 + 16 i + 4 j + k."""
    s = np.asarray(scales, dtype=np.uint8)
    rows, C = s.shape
    rows_pad, C_pad = -(-rows // 128) * 128, -(-C // 4) * 4
    full = np.zeros((rows_pad, C_pad), np.uint8)
    full[:rows, :C] = s
    # [r][j][i][c][k] -> [r][c][i][j][k]
    t = full.reshape(rows_pad // 128, 4, 32, C_pad // 4, 4)
    return np.ascontiguousarray(t.transpose(0, 3, 2, 1, 4)).reshape(-1)


def gemm_mx(a_codes: np.ndarray, a_scales: np.ndarray, b_codes: np.ndarray, b_scales: np.ndarray) -> np.ndarray:
    """The FP4 MatMul after WUSH + Quant ([graph] §3.4.7 "GPU Kernel Design": the
    transformed, quantised activations multiply the pre-quantised weights):
    D = deq(A) deq(B)^T in float64, A packed MXFP4 codes [M][K/2] with scales [M][K/32],
    B packed codes [N][K/2] with scales [N][K/32] (one row per output channel)."""
    A = dequant(unpack_nibbles(a_codes), a_scales, "mxfp4", 32)
    B = dequant(unpack_nibbles(b_codes), b_scales, "mxfp4", 32)
    return A @ B.T


def gemm_nv(a_codes: np.ndarray, a_scales: np.ndarray, a_ts: float, b_codes: np.ndarray, b_scales: np.ndarray,
            b_ts: float) -> np.ndarray:
    """The same product for NVFP4 operands (E4M3 scales per 16 elements [rows][K/16] and
    an fp32 tensor scale each): D = deq(A) deq(B)^T in float64."""
    A = dequant(unpack_nibbles(a_codes), a_scales, "nvfp4", 16, a_ts)
    B = dequant(unpack_nibbles(b_codes), b_scales, "nvfp4", 16, b_ts)
    return A @ B.T


def grid_step_distance(ca: np.ndarray, cb: np.ndarray, fmt: str) -> np.ndarray:
    """Number of grid steps between two code arrays of the same scale, counting
    the step through zero (+0.5 <-> 0 <-> -0.5 for E2M1; +1 <-> 0 <-> -1 for INT4)."""
    if fmt in ("mxfp4", "nvfp4"):
        def pos(c):
            c = np.asarray(c, dtype=np.int64)
            m = c & 7
            return np.where(c & 8, -m, m)
    else:
        def pos(c):
            return int4_decode(c).astype(np.int64)
    return np.abs(pos(ca) - pos(cb))
