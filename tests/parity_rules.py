"""GPU-vs-oracle comparison rules used by the GPU tests.

Rule 1 (bit-exact): the oracle quantiser fed the kernel's own fp32 transformed
values must reproduce the kernel's codes and scales exactly (E2M1 codes 0x0 and 0x8
both mean zero and compare equal).

Rule 2 (end to end): the oracle's float64 path on the same inputs; dequantised
outputs agree within a relative Frobenius error of 2e-3, and at most 0.1 % of the
codes differ, each by one grid step.  A group whose scale differs counts in full
toward the 0.1 %, and each of its elements must lie within one grid step at the
finer of the two scales.  INT4 scales are fp32 values (amax / 7), so "the same scale"
there means equal within a relative 2^-14, the precision of the kernel's fp32 y.
"""
from __future__ import annotations

import numpy as np

from oracle import wush_oracle as O

REL_FROB_TOL = 2e-3
FLIP_FRAC_TOL = 1e-3
INT4_SCALE_RTOL = 2.0 ** -14


def canon_codes(codes: np.ndarray, fmt: str, packed: bool = False) -> np.ndarray:
    """Unpacked codes with negative zero (E2M1 0x8) folded onto 0x0."""
    c = O.unpack_nibbles(codes) if packed else np.asarray(codes)
    if fmt in ("mxfp4", "nvfp4"):
        c = np.where(c == 8, 0, c).astype(np.uint8)
    return c


def oracle_quantize(y, fmt, G, s_t=None):
    """The oracle quantiser; for NVFP4 an explicit tensor scale replaces the one taken
    from max |y| (used when y holds only sampled groups of a larger tensor)."""
    y = np.asarray(y, dtype=np.float64)
    if fmt == "nvfp4" and s_t is not None:
        return O.quant_nvfp4(y, float(s_t))
    return O.quantize(y, fmt, G)


def assert_bit_exact(codes_gpu, scales_gpu, ts_gpu, y_gpu, fmt, G, s_t=None):
    """Rule 1.  ``s_t``: the oracle's NVFP4 tensor scale when y is a sample."""
    c_o, s_o, ts_o = oracle_quantize(y_gpu, fmt, G, s_t)
    c_g = canon_codes(codes_gpu, fmt, packed=True)
    c_o = canon_codes(c_o, fmt)
    if fmt == "nvfp4":
        assert np.float32(ts_gpu) == np.float32(ts_o), (ts_gpu, ts_o)
    bad_s = np.argwhere(np.asarray(scales_gpu) != np.asarray(s_o))
    assert bad_s.size == 0, f"{len(bad_s)} scales differ, first at {bad_s[:5].tolist()}: " \
                            f"gpu {np.asarray(scales_gpu)[tuple(bad_s[0])]} oracle {np.asarray(s_o)[tuple(bad_s[0])]}"
    bad = np.argwhere(c_g != c_o)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:5].tolist()}: " \
                          f"gpu {c_g[tuple(bad[0])]} oracle {c_o[tuple(bad[0])]} y {y_gpu[tuple(bad[0])]}"


def group_scale_values(scales, fmt, G, ts):
    s = np.asarray(scales)
    if fmt == "mxfp4":
        return np.exp2(s.astype(np.float64) - 127.0)
    if fmt == "nvfp4":
        return O.e4m3_decode(s) * float(ts)
    return s.astype(np.float64)


def end_to_end_report(codes_gpu, scales_gpu, ts_gpu, y_ref, fmt, G, s_t_ref=None):
    """Rule 2 statistics: (rel_frob, flip_fraction, n_scale_groups_differing, max_steps).
    ``s_t_ref``: the oracle's NVFP4 tensor scale when y_ref is a sample."""
    c_o, s_o, ts_o = oracle_quantize(y_ref, fmt, G, s_t_ref)
    c_g = O.unpack_nibbles(codes_gpu)
    n, d = c_g.shape
    deq_g = O.dequant(c_g, scales_gpu, fmt, G, ts_gpu)
    deq_o = O.dequant(c_o, s_o, fmt, G, ts_o)
    denom = np.linalg.norm(deq_o)
    rel = float(np.linalg.norm(deq_g - deq_o) / denom) if denom > 0 else float(np.linalg.norm(deq_g))
    if fmt == "int4":
        # fp32 scales amax/7 inherit the fp32-vs-fp64 rounding of y: equal within 2^-14
        sg, so = np.asarray(scales_gpu, np.float64), np.asarray(s_o, np.float64)
        same_scale = np.abs(sg - so) <= INT4_SCALE_RTOL * so
    else:
        same_scale = (np.asarray(scales_gpu) == np.asarray(s_o))              # [n][C]
    steps = O.grid_step_distance(c_g, c_o, fmt).reshape(n, d // G, G)
    diff_in_same = (steps > 0) & same_scale[:, :, None]
    max_steps_same = int(steps[same_scale].max()) if same_scale.any() and steps.size else 0
    n_scale_diff = int((~same_scale).sum())
    flips = int(diff_in_same.sum()) + n_scale_diff * G
    # groups whose scale differs: each element within one grid step at the finer scale
    if n_scale_diff:
        sg = group_scale_values(scales_gpu, fmt, G, ts_gpu)
        so = group_scale_values(s_o, fmt, G, ts_o)
        finer = np.minimum(sg, so)[:, :, None]
        max_step_units = 2.0 if fmt in ("mxfp4", "nvfp4") else 1.0
        dg = deq_g.reshape(n, d // G, G)
        do = deq_o.reshape(n, d // G, G)
        mask = ~same_scale
        ok = np.abs(dg - do)[mask] <= (max_step_units * finer)[mask] * (1 + 1e-6)
        assert ok.all(), "a group with a differing scale is off by more than one grid step"
    return rel, flips / float(n * d), n_scale_diff, max_steps_same


def assert_end_to_end(codes_gpu, scales_gpu, ts_gpu, y_ref, fmt, G, s_t_ref=None):
    rel, frac, nsd, mx = end_to_end_report(codes_gpu, scales_gpu, ts_gpu, y_ref, fmt, G, s_t_ref)
    assert mx <= 1, f"a code differs by {mx} grid steps"
    assert rel <= REL_FROB_TOL, f"relative Frobenius error {rel:.3e} > {REL_FROB_TOL}"
    assert frac <= FLIP_FRAC_TOL, f"{frac:.3e} of codes differ (> {FLIP_FRAC_TOL}); {nsd} groups differ in scale"
    return rel, frac, nsd
