"""Layerwise-loss harness on synthetic layers.

Mirrors the structure of the pages' per-layer loss table (paper-graph-ui analysis,
section 5 "Per-Layer Quantization Loss (Table 1)"; the loss is the normalised
Frobenius error of section 3.4.1, Eq. (5)) without models or datasets: one synthetic
linear layer (weights W, calibration activations X_cal and held-out activations X from
the seeded workload generator) is quantised under every transform

  I     identity,
  R     a random orthogonal matrix per block (averaged over several draws),
  H     the normalised Hadamard matrix in every block,
  WUS   the WUSH construction without its Hadamard factor,
  WUSH  the full construction,

and every format (MXFP4 G=32, NVFP4 G=16, INT4 G=32), with RTN AbsMax quantisation on
the GPU (wush_quant_act / wush_quant_weight), dequantisation (wush_dequant), and

  L = || W^T X - q(T_W W)^T q(T_X X) ||_F^2 / (d_out d_batch)

from float64 GEMMs of the dequantised operands.  Activations take T_wush and weights
T_xvsh (for the orthogonal transforms both are the same matrix).  As in the pages, the
loss is reported on the calibration tokens the transforms were built from; the loss
on held-out tokens is reported beside it.

    python -m blockwise_adaptive_transforms_b200.loss_harness --workload attn_mxfp4_4096
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np
import torch

from . import (wush_hadamard, wush_build_transforms, wush_dequant, wush_quant_act,
               wush_quant_weight)

FORMATS = (("mxfp4", 32), ("nvfp4", 16), ("int4", 32))
KINDS = ("I", "R", "H", "WUS", "WUSH")


def random_orthogonal_blocks(C: int, G: int, seed: int, device) -> torch.Tensor:
    """C random orthogonal G x G matrices (QR of a Gaussian draw, signs fixed by R's
    diagonal so the draw is Haar-distributed), fp32 [C][G][G]."""
    rng = np.random.default_rng(seed)
    q, r = np.linalg.qr(rng.standard_normal((C, G, G)))
    q = q * np.sign(np.diagonal(r, axis1=1, axis2=2))[:, None, :]
    return torch.from_numpy(q.astype(np.float32)).to(device)


def layer_loss(w: torch.Tensor, x: torch.Tensor, T_act: torch.Tensor, T_weight: torch.Tensor,
               G: int, fmt: str, ref: torch.Tensor | None = None) -> float:
    """Normalised Frobenius loss of one quantised layer.

    w: fp32 [d_out][d_in] (row = output channel); x: bf16 [n][d_in] (row = token);
    T_act, T_weight: fp32 [C][G][G].  ``ref`` (optional) is W^T X in float64."""
    cw, sw, tw = wush_quant_weight(w, T_weight, G, fmt)
    cx, sx, tx = wush_quant_act(x, T_act, G, fmt)
    wq = wush_dequant(cw, sw, tw, G, fmt).double()
    xq = wush_dequant(cx, sx, tx, G, fmt).double()
    if ref is None:
        ref = w.double() @ x.double().T
    err = ref - wq @ xq.T
    return float((err * err).mean())


def transforms(kind: str, w: torch.Tensor, xcal: torch.Tensor, G: int, seed: int = 0):
    """(T_act, T_weight) for one transform kind, fp32 [C][G][G] on w's device."""
    C = w.shape[1] // G
    dev = w.device
    if kind == "I":
        T = torch.eye(G, device=dev).repeat(C, 1, 1).contiguous()
        return T, T
    if kind == "H":
        T = wush_hadamard(G, copies=C, device=dev)
        return T, T
    if kind == "R":
        T = random_orthogonal_blocks(C, G, seed, dev)
        return T, T
    if kind in ("WUS", "WUSH"):
        T_wush, T_xvsh = wush_build_transforms(w, xcal, G, use_hadamard=(kind == "WUSH"))
        return T_wush, T_xvsh
    raise ValueError(kind)


def loss_table(workload_name: str, eval_tokens: int | None = None, rand_runs: int = 10,
               kinds=KINDS, formats=FORMATS, device="cuda") -> dict:
    """Loss of every (format, transform) pair on one synthetic layer (the same W, X_cal
    and X for every format; the transforms are built per group size)."""
    from workloads import make_inputs, workload

    wl = workload(workload_name)
    inp = make_inputs(wl, n_tok=eval_tokens)
    w = torch.from_numpy(inp.w).to(device)
    xcal = torch.from_numpy(inp.xcal_bits.view(np.int16)).view(torch.bfloat16).to(device)
    xev = torch.from_numpy(inp.x_bits.view(np.int16)).view(torch.bfloat16).to(device)
    ref_cal = w.double() @ xcal.double().T
    ref_ev = w.double() @ xev.double().T
    msq = float((ref_cal * ref_cal).mean())
    out = {"workload": workload_name,
           "shape": {"d_in": wl.d_in, "d_out": wl.d_out, "calibration_tokens": int(xcal.shape[0]),
                     "heldout_tokens": int(xev.shape[0])},
           "loss": {}, "loss_heldout": {}, "rel": {}}
    for fmt, G in formats:
        row, row_ev, row_rel = {}, {}, {}
        for kind in kinds:
            runs = rand_runs if kind == "R" else 1
            l_cal = l_ev = 0.0
            for r in range(runs):
                T_act, T_weight = transforms(kind, w, xcal, G, seed=r)
                l_cal += layer_loss(w, xcal, T_act, T_weight, G, fmt, ref_cal) / runs
                l_ev += layer_loss(w, xev, T_act, T_weight, G, fmt, ref_ev) / runs
            row[kind], row_ev[kind], row_rel[kind] = l_cal, l_ev, l_cal / msq
        out["loss"][fmt], out["loss_heldout"][fmt], out["rel"][fmt] = row, row_ev, row_rel
    return out


def format_table(res: dict) -> str:
    kinds = list(next(iter(res["loss"].values())).keys())
    lines = [f"layerwise RTN loss, {res['workload']} {res['shape']}",
             "format   " + "".join(f"{k:>12s}" for k in kinds)]
    for fmt, row in res["loss"].items():
        lines.append(f"{fmt:8s} " + "".join(f"{row[k]:12.4g}" for k in kinds))
    lines.append("relative to mean (W^T X)^2:")
    for fmt, row in res["rel"].items():
        lines.append(f"{fmt:8s} " + "".join(f"{row[k]:12.4g}" for k in kinds))
    return "\n".join(lines)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="attn_mxfp4_4096")
    ap.add_argument("--eval-tokens", type=int, default=2048)
    ap.add_argument("--rand-runs", type=int, default=10)
    ap.add_argument("--json", default=None, help="also write the table as JSON here")
    a = ap.parse_args(argv)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    res = loss_table(a.workload, a.eval_tokens, a.rand_runs)
    print(format_table(res))
    if a.json:
        with open(a.json, "w") as f:
            json.dump(res, f, indent=1)
    return 0


if __name__ == "__main__":
    sys.exit(main())
