"""Seeded synthetic inputs for the fused blockwise-transform + 4-bit quantisation path.

This module draws random numbers and nothing else: it holds none of the method's
arithmetic (no second moments, no factorisations, no transform, no quantiser).
Both the CUDA path's tests/benchmark and the independent oracle take their
inputs from here, so that the two sides see the same bytes.

Value model (one per workload, see ``WORKLOADS``): for every token a base vector
z is drawn (normal, Student-t(4) or Laplace), each block of G channels is mixed
by its own random lower-triangular matrix L_i (diagonal ~ U[0.5, 2], strictly
lower entries ~ N(0, 1/G)), then every channel j is multiplied by a channel scale
c_j (log-normal(0, 1) where the workload asks for it, else 1) and, for the
outlier channels, by the outlier multiplier.  The calibration activations use the
same L_i, channel scales and outlier set with a separate draw of z.

Random streams: ``numpy.random.default_rng`` (PCG64) seeded from
``SeedSequence(seed).spawn(6)``; streams 0..5 are, in order: outlier channel set,
mixing matrices L_i, channel scales, calibration tokens, timed activations X,
weights W.  Values are generated in float64 and rounded once: activations to
bfloat16 (float64 -> float32 round-to-nearest-even, then float32 -> bfloat16
round-to-nearest-even on the bit pattern), weights to float32.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "bf16_bits_from_f64", "bf16_bits_to_f32",
           "make_inputs", "Inputs"]


@dataclass(frozen=True)
class Workload:
    name: str
    n_tok: int          # timed activation rows (tokens)
    d_in: int           # input channels
    G: int              # block size = quantisation group size
    fmt: str            # "mxfp4" | "nvfp4" | "int4"
    d_out: int          # output channels of the weight matrix
    n_cal: int          # calibration tokens used to build the transforms
    base: str           # "normal" | "student_t4" | "laplace"
    lognormal_scales: bool
    n_outliers: int     # number of outlier channels
    outlier_mult: float
    seed: int


# The five workloads: tiny MXFP4, Llama-8B-like attention input (MXFP4),
# MLP down-projection (NVFP4), 70B-like large batch (MXFP4) and the INT4 token sweep.
WORKLOADS = {
    "tiny_mxfp4": Workload("tiny_mxfp4", 64, 256, 32, "mxfp4", 128, 512,
                           "normal", False, 2, 20.0, 0),
    "attn_mxfp4_4096": Workload("attn_mxfp4_4096", 4096, 4096, 32, "mxfp4", 4096, 2048,
                                "normal", True, 20, 30.0, 2),
    "mlp_down_nvfp4_14336": Workload("mlp_down_nvfp4_14336", 4096, 14336, 16, "nvfp4", 4096, 2048,
                                     "student_t4", False, 143, 50.0, 3),
    "large_mxfp4_8192": Workload("large_mxfp4_8192", 16384, 8192, 32, "mxfp4", 8192, 2048,
                                 "normal", True, 41, 30.0, 4),
    "int4_sweep_4096": Workload("int4_sweep_4096", 8192, 4096, 32, "int4", 4096, 2048,
                                "laplace", False, 0, 1.0, 5),
}
INT4_SWEEP_TOKENS = (1, 16, 128, 1024, 8192)


def workload(name: str, **overrides) -> Workload:
    """Return a named workload, optionally with fields replaced (e.g. a smaller n_tok)."""
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def bf16_bits_from_f64(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 and return the 16-bit patterns (uint16).

    float64 -> float32 uses numpy's round-to-nearest-even cast; float32 -> bfloat16
    adds 0x7FFF plus the lowest kept bit and truncates (round-to-nearest-even).
    Inputs are finite by construction.
    """
    f = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (f >> np.uint32(16)) & np.uint32(1)
    return ((f + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Inputs:
    wl: Workload
    x_bits: np.ndarray      # uint16 [n_tok][d_in]  bfloat16 activations
    xcal_bits: np.ndarray   # uint16 [n_cal][d_in]  bfloat16 calibration activations
    w: np.ndarray           # float32 [d_out][d_in] weights (one row per output channel)


def _base_draw(rng: np.random.Generator, base: str, shape) -> np.ndarray:
    if base == "normal":
        return rng.standard_normal(shape)
    if base == "student_t4":
        return rng.standard_t(4.0, shape)
    if base == "laplace":
        return rng.laplace(0.0, 1.0, shape)
    raise ValueError(base)


def _activations(rng, wl: Workload, n: int, L: np.ndarray, chan: np.ndarray,
                 chunk: int = 2048) -> np.ndarray:
    """Draw n tokens of the workload's value model; returns bfloat16 bits [n][d_in]."""
    C, G = wl.d_in // wl.G, wl.G
    out = np.empty((n, wl.d_in), dtype=np.uint16)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        z = _base_draw(rng, wl.base, (r1 - r0, C, G))
        u = np.einsum("cij,ncj->nci", L, z).reshape(r1 - r0, wl.d_in)
        out[r0:r1] = bf16_bits_from_f64(u * chan[None, :])
    return out


def make_inputs(wl: Workload, n_tok: int | None = None, need_w: bool = True,
                need_cal: bool = True) -> Inputs:
    """Generate the workload's activations, calibration activations and weights.

    ``n_tok`` overrides the number of timed tokens (the first n_tok rows of the
    full draw are returned unchanged, because the draw is chunked by rows).
    """
    if wl.d_in % wl.G:
        raise ValueError("d_in must be a multiple of G")
    C, G = wl.d_in // wl.G, wl.G
    ss = np.random.SeedSequence(wl.seed).spawn(6)
    r_out, r_mix, r_scale, r_cal, r_x, r_w = (np.random.default_rng(s) for s in ss)

    mult = np.ones(wl.d_in)
    if wl.n_outliers:
        idx = r_out.choice(wl.d_in, size=wl.n_outliers, replace=False)
        mult[idx] = wl.outlier_mult
    L = np.tril(r_mix.standard_normal((C, G, G)) / np.sqrt(G), -1)
    L[:, np.arange(G), np.arange(G)] = r_mix.uniform(0.5, 2.0, (C, G))
    scales = r_scale.lognormal(0.0, 1.0, wl.d_in) if wl.lognormal_scales else np.ones(wl.d_in)
    chan = scales * mult

    n = wl.n_tok if n_tok is None else int(n_tok)
    xcal = _activations(r_cal, wl, wl.n_cal, L, chan) if need_cal else np.zeros((0, wl.d_in), np.uint16)
    x = _activations(r_x, wl, n, L, chan)
    if need_w:
        w = (r_w.standard_normal((wl.d_out, wl.d_in)) / np.sqrt(wl.d_in)).astype(np.float32)
    else:
        w = np.zeros((0, wl.d_in), np.float32)
    return Inputs(wl, x, xcal, w)
