"""Per-layer speedup of the quantised FP4 layer over the bf16 layer.

Mirrors the pages' kernel benchmark (paper-graph-ui analysis, section 5 "GPU Kernel
Benchmarks (Figure 2)": per-layer MXFP4 GEMM speedup relative to BF16 at batch M = 1024,
for a square, a wide and a deep projection of each model) on one B200:

  bf16   X W^T in bf16 (cuBLAS through torch.matmul),
  none   the MXFP4 GEMM alone, operands already quantised (the upper bound),
  H      shared-Hadamard transform + quantisation of X, then the MXFP4 GEMM,
  WUSH   per-block WUSH transform + quantisation of X, then the MXFP4 GEMM;
  nv_none / nv_WUSH   the same two for NVFP4 (G = 16 transforms, two-pass tensor scale
         in one cooperative launch, the NVFP4 GEMM); nv_WUSH_4launch the same layer with
         the activation quantiser's four launches.

Weights are quantised once beforehand (offline, as on the pages).  Every variant is
timed as a CUDA graph of repeated calls with events on its stream.

    python -m blockwise_adaptive_transforms_b200.layer_bench [--shapes qwen3-8b]
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

from . import (nvfp4_workspace, wush_hadamard, wush_gemm_mxfp4, wush_gemm_nvfp4, wush_quant_act_mx_atoms,
               wush_quant_act_nv_atoms, wush_quant_act_nv_atoms_onepass, wush_quant_act_shared_mx_atoms,
               wush_quant_weight_mx_atoms, wush_quant_weight_nv_atoms)

# (N, K) per projection kind.  The Qwen3-8B shapes are the pages' own; the other two rows
# are the same three kinds for a 14B-class (hidden 5120, MLP 17408) and a 70B-class
# (hidden 8192, MLP 28672) model.
SHAPES = {
    "qwen3-8b": [(4096, 4096), (24576, 4096), (4096, 12288)],
    "14b-class": [(5120, 5120), (34816, 5120), (5120, 17408)],
    "70b-class": [(8192, 8192), (57344, 8192), (8192, 28672)],
}


def _time_graph(fn, stream, iters=50, reps=5) -> float:
    """Best-of-reps microseconds per call of fn, replayed from a CUDA graph."""
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(iters):
                fn()
        g.replay()
        stream.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1) * 1e3 / iters)
    del g
    return best


def bench_shape(M: int, N: int, K: int, device="cuda", seed=0) -> dict:
    gen = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(M, K, generator=gen).to(torch.bfloat16).to(device)
    w = (torch.randn(N, K, generator=gen) / K ** 0.5).to(device)
    C = K // 32
    T = (torch.eye(32) + 0.1 * torch.randn(C, 32, 32, generator=gen)).to(device)
    H = wush_hadamard(32, device=device)
    w_bf16 = w.to(torch.bfloat16)
    cw, aw = wush_quant_weight_mx_atoms(w, T)             # offline
    cx, ax = wush_quant_act_mx_atoms(x, T)
    Tn = (torch.eye(16) + 0.1 * torch.randn(K // 16, 16, 16, generator=gen)).to(device)
    cwn, awn, twn = wush_quant_weight_nv_atoms(w, Tn)     # offline
    cxn, axn, txn = wush_quant_act_nv_atoms(x, Tn)
    ws = nvfp4_workspace(device=device)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    out_ref = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    s = torch.cuda.Stream(device=device)

    def bf16():
        torch.matmul(x, w_bf16.T, out=out_ref)

    def none():
        wush_gemm_mxfp4(cx, ax, cw, aw, out=out, stream=s)

    def h_quant():
        wush_quant_act_shared_mx_atoms(x, H, codes=cx, atoms=ax, stream=s)
        wush_gemm_mxfp4(cx, ax, cw, aw, out=out, stream=s)

    def wush():
        wush_quant_act_mx_atoms(x, T, codes=cx, atoms=ax, stream=s)
        wush_gemm_mxfp4(cx, ax, cw, aw, out=out, stream=s)

    def nv_none():
        wush_gemm_nvfp4(cxn, axn, txn, cwn, awn, twn, out=out, stream=s)

    def nv_wush():   # the two-pass quantiser in one launch
        wush_quant_act_nv_atoms_onepass(x, Tn, ws, codes=cxn, atoms=axn, tensor_scale=txn, stream=s)
        wush_gemm_nvfp4(cxn, axn, txn, cwn, awn, twn, out=out, stream=s)

    def nv_wush4():   # the same in four launches
        wush_quant_act_nv_atoms(x, Tn, codes=cxn, atoms=axn, tensor_scale=txn, stream=s)
        wush_gemm_nvfp4(cxn, axn, txn, cwn, awn, twn, out=out, stream=s)

    t = {name: _time_graph(fn, s) for name, fn in (("bf16", bf16), ("none", none), ("H", h_quant), ("WUSH", wush),
                                                   ("nv_none", nv_none), ("nv_WUSH", nv_wush),
                                                   ("nv_WUSH_4launch", nv_wush4))}
    flops = 2.0 * M * N * K
    return {"M": M, "N": N, "K": K, "us": {k: round(v, 2) for k, v in t.items()},
            "speedup_vs_bf16": {k: round(t["bf16"] / t[k], 3)
                                for k in ("none", "H", "WUSH", "nv_none", "nv_WUSH", "nv_WUSH_4launch")},
            "fp4_gemm_tflops": round(flops / t["none"] / 1e6, 1), "bf16_tflops": round(flops / t["bf16"] / 1e6, 1)}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--shapes", default=",".join(SHAPES), help="comma-separated keys of SHAPES")
    ap.add_argument("--M", type=int, default=1024)
    ap.add_argument("--json", default=None)
    a = ap.parse_args(argv)
    rows = []
    for key in a.shapes.split(","):
        for N, K in SHAPES[key]:
            r = bench_shape(a.M, N, K)
            r["model"] = key
            rows.append(r)
            print(f"{key:10s} M={a.M} N={N:6d} K={K:6d}  bf16 {r['us']['bf16']:8.1f} us  fp4 gemm {r['us']['none']:8.1f} us"
                  f" ({r['fp4_gemm_tflops']:7.1f} TFLOP/s)  H {r['us']['H']:8.1f}  WUSH {r['us']['WUSH']:8.1f}   "
                  f"speedup none/H/WUSH {r['speedup_vs_bf16']['none']:.2f}/{r['speedup_vs_bf16']['H']:.2f}/"
                  f"{r['speedup_vs_bf16']['WUSH']:.2f}   nvfp4 none/WUSH {r['us']['nv_none']:8.1f}/{r['us']['nv_WUSH']:8.1f} us"
                  f" (4 launches {r['us']['nv_WUSH_4launch']:8.1f})",
                  flush=True)
    if a.json:
        with open(a.json, "w") as f:
            json.dump(rows, f, indent=1)
    return 0


if __name__ == "__main__":
    sys.exit(main())
