"""Run one quantiser configuration a few times, for a profiler to capture.

``python -m blockwise_adaptive_transforms_b200.profile_case --fmt mxfp4 --rows 16384 --d-in 8192``
quantises seeded bf16 activations (near-identity per-block transforms) ``--launches``
times on one stream, after ``--warmup`` untimed calls, and checks the device error word.
``--sets N`` rotates over N input/output sets, so that, as in the benchmark, each call
reads its input from DRAM and the previous calls' outputs are written back while it runs.
Use ``ncu -k regex:wush_fused_kernel -s <warmup launches>`` to capture the timed calls.
``--one-launch`` (NVFP4 only) makes every call after the first set's outputs one
cooperative launch (wush_quant_act_nvfp4_onepass) instead of four.
"""
from __future__ import annotations

import argparse

import torch

import blockwise_adaptive_transforms_b200 as W

GROUP = {"mxfp4": 32, "nvfp4": 16, "int4": 32}


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--fmt", choices=sorted(GROUP), default="mxfp4")
    ap.add_argument("--rows", type=int, default=16384)
    ap.add_argument("--d-in", type=int, default=8192)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--launches", type=int, default=2)
    ap.add_argument("--sets", type=int, default=1)
    ap.add_argument("--one-launch", action="store_true")
    args = ap.parse_args(argv)
    if args.one_launch and args.fmt != "nvfp4":
        raise SystemExit("--one-launch applies to nvfp4 only")
    G = GROUP[args.fmt]
    C = args.d_in // G
    g = torch.Generator().manual_seed(0)
    xs = [torch.randn(args.rows, args.d_in, generator=g).to(torch.bfloat16).cuda() for _ in range(args.sets)]
    T = (torch.eye(G).repeat(C, 1, 1) + 0.05 * torch.randn(C, G, G, generator=g)).float().cuda()
    outs = [W.wush_quant_act(x, T, G, args.fmt) for x in xs]
    ws = W.nvfp4_workspace() if args.one_launch else None
    for i in range(args.sets, args.warmup + args.launches):
        k = i % args.sets
        if args.one_launch:
            W.wush_quant_act_nvfp4_onepass(xs[k], T, ws, codes=outs[k][0], scales=outs[k][1],
                                           tensor_scale=outs[k][2])
        else:
            W.wush_quant_act(xs[k], T, G, args.fmt, codes=outs[k][0], scales=outs[k][1],
                             tensor_scale=outs[k][2])
    torch.cuda.synchronize()
    st, bits = W.wush_device_status()
    if st != 0:
        raise SystemExit(f"device error word {bits:#x}")
    print(f"ok: {args.fmt} {args.rows} x {args.d_in}, {args.warmup + args.launches} calls")


if __name__ == "__main__":
    main()
