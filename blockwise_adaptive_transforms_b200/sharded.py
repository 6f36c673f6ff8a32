"""NVFP4 activations of a batch whose token rows are split across ranks (one process per
GPU, torch.distributed; NCCL over NVLink between GPUs).

NVFP4 scales each 16-value group by an E4M3 factor under one fp32 tensor scale, and the
tensor scale is fixed by the AbsMax of the whole tensor (s_t = amax / (6 * 448): the
NVFP4 two-level scale the pages name in paper-graph-ui analysis, section 3.4.1; the pages
do not say how s_t is obtained, and a global AbsMax is the plain reading).  When the
batch's rows live on several ranks, the per-rank amax values must meet before any rank
quantises: the one exchange of the path, a max all-reduce of a single fp32 between the
amax pass and the quantising pass.  MXFP4 and INT4 scales are per group, so their shards
need no exchange at all.

    codes, scales, s_t = quant_act_nvfp4_sharded(x_local, T_wush16, group)

Every rank gets the same s_t, and its codes and scales are what the single-device call
would produce for its rows of the full batch.
"""
from __future__ import annotations

import contextlib

import torch
import torch.distributed as dist

from . import wush_nvfp4_scale_from_amax, wush_quant_act_nvfp4_amax, wush_quant_act_nvfp4_with_scale

__all__ = ["quant_act_nvfp4_sharded"]

# The three device stages, looked up at call time (a CPU test of the rank logic swaps in
# host stand-ins; the binding itself only accepts CUDA tensors).
_stages = {"amax": wush_quant_act_nvfp4_amax, "scale": wush_nvfp4_scale_from_amax,
           "quantise": wush_quant_act_nvfp4_with_scale}


def quant_act_nvfp4_sharded(x, T, group=None, stream=None, codes=None, scales=None):
    """x: this rank's bf16 rows [n_local][d_in]; T: fp32 [d_in/16][16][16].
    Returns (codes [n_local][d_in/2], E4M3 scales [n_local][d_in/16], tensor scale [1])."""
    if x.is_cuda:
        s = stream if stream is not None else torch.cuda.current_stream(x.device)
        ctx = torch.cuda.stream(s)
    else:
        s, ctx = stream, contextlib.nullcontext()
    with ctx:
        amax = _stages["amax"](x, T, stream=s)
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
        _stages["scale"](amax, stream=s)
        codes, scales = _stages["quantise"](x, T, amax, codes=codes, scales=scales, stream=s)
    return codes, scales, amax
