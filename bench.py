#!/usr/bin/env python
"""Throughput of the fused WUSH transform + MXFP4 quantisation on the Llama-8B-like
attention-input workload: 4096 tokens x d_in = 4096, G = 32, bf16 activations.

One step = one call of wush_quant_act over the whole 4096 x 4096 batch.  Inputs are
resident in HBM; eight rotating input/output sets (8 x 43 MB > 126 MB L2) make every
step read its activations from DRAM.  The timed region is nine spans, each bracketed
by a barrier + synchronize and CUDA events on the launching stream, each replaying a
CUDA graph of back-to-back launches max(K, 4000) times over; the median span gives
the time per step, so the figure does not depend on how small K is.  Under torchrun
every rank runs its own batch (weak scaling) and each span's time is the maximum over
ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line (rank 0).  ``--impl reference`` times the float64 CPU oracle on
the host cores instead, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "WUSH+quant GB/s & tokens/s at d=4096 G=32 MXFP4; % of HBM roofline"
WORKLOAD = "attn_mxfp4_4096"
N_SETS = 8
GRAPH_LEN = 1000         # launches per captured graph
SPAN_MIN_LAUNCHES = 4000   # launches per timed span (about 40 ms at this size)
N_SPANS = 9              # timed spans; the median is reported
FALLBACK_HBM_GBS = 6650.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "wush_fused_mxfp4_attn_4096.md")
KERNEL_SOURCES = ("blockwise_adaptive_transforms_b200/csrc/wush_fused.cuh",
                  "blockwise_adaptive_transforms_b200/csrc/wush_ptx.cuh")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--span-launches", type=int, default=SPAN_MIN_LAUNCHES,
                    help="least launches per timed span (a short value suits profiler runs)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true",
                    help="skip the per-configuration rows (NVFP4, large batch, weights, INT4 sweep, FP4 GEMM)")
    return ap.parse_args()


def algorithmic_bytes(n_tok: int, d_in: int, G: int) -> int:
    """Bytes one step must move: read x (bf16) and T (fp32), write codes and E8M0 scales."""
    C = d_in // G
    return n_tok * d_in * 2 + n_tok * d_in // 2 + n_tok * C + C * G * G * 4


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over all ranks (the timing rule: the slowest rank decides)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, bytes_per_step: int, elapsed_s: float) -> float:
    """Whole-job GB/s: every rank processes its own batch per step (weak scaling)."""
    return world * steps * bytes_per_step / elapsed_s / 1e9


def _code_only(text: str) -> str:
    """The source without comments and blank lines: what the compiled kernel depends on."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash() -> str:
    """SHA-256 (16 hex digits) of the fused kernel's sources, comments excluded."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source; else None."""
    try:
        fields = {}
        with open(PROFILE_SUMMARY) as f:
            for line in f:
                if ":" in line and line.strip().startswith("- "):
                    k, v = line.strip()[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if fields.get("kernel_source_sha256_16") != kernel_source_hash():
            return None
        return int(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running (read only)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                import torch
                p = torch.cuda.get_device_properties(device_index)
                bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def _oracle_pool_init(root: str) -> None:
    """Worker set-up: one thread per worker process (the pool supplies the parallelism)."""
    for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[k] = "1"
    if root not in sys.path:
        sys.path.insert(0, root)


def _oracle_slice(task) -> int:
    """One bounded sample for a pool worker: the oracle's whole path on a row slice."""
    x_bits, T32, G, fmt = task
    from oracle import wush_oracle as O
    O.quant_act(x_bits, T32, G, fmt)
    return int(x_bits.shape[0])


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_pool(n: int):
    """A process pool of n oracle workers, started with spawn (safe after CUDA is up)."""
    import multiprocessing as mp
    return mp.get_context("spawn").Pool(n, initializer=_oracle_pool_init, initargs=(ROOT,))


def _slices(x_bits, rows: int, k0: int, n: int):
    n_tok = x_bits.shape[0]
    return [x_bits[((k0 + j) * rows) % n_tok:((k0 + j) * rows) % n_tok + rows] for j in range(n)]


def cpu_baseline(inp, wl, seconds: float):
    """The float64 oracle, as it stands, on the host cores: 256-token samples of the
    workload, on all cores (one worker process per core, each running the oracle on its
    own slice) and on one core, about `seconds` each, scaled to the metric's bytes."""
    from oracle import wush_oracle as O
    from threadpoolctl import threadpool_limits
    b = O.build_transforms(inp.w, inp.xcal_bits, wl.G)
    T32 = b["T_wush32"]
    rows = 256
    per_tok = algorithmic_bytes(wl.n_tok, wl.d_in, wl.G) / wl.n_tok
    # one core
    with threadpool_limits(limits=1):
        O.quant_act(inp.x_bits[:rows], T32, wl.G, wl.fmt)
        done1, t1, j = 0, time.perf_counter(), 0
        while time.perf_counter() - t1 < seconds:
            done1 += _oracle_slice((_slices(inp.x_bits, rows, j, 1)[0], T32, wl.G, wl.fmt))
            j += 1
        dt1 = time.perf_counter() - t1
    # every core: one slice per worker per round
    n = host_cores()
    with oracle_pool(n) as pool:
        pool.map(_oracle_slice, [(x, T32, wl.G, wl.fmt) for x in _slices(inp.x_bits, rows, 0, n)])
        done, t0, k = 0, time.perf_counter(), 0
        while time.perf_counter() - t0 < seconds:
            done += sum(pool.map(_oracle_slice, [(x, T32, wl.G, wl.fmt) for x in _slices(inp.x_bits, rows, k, n)]))
            k += n
        dt = time.perf_counter() - t0
    return {"value": round(done / dt * per_tok / 1e9, 6), "unit": "GB/s", "cores": n, "kind": "oracle",
            "tokens_per_s": round(done / dt, 1),
            "one_core": {"value": round(done1 / dt1 * per_tok / 1e9, 6), "tokens_per_s": round(done1 / dt1, 1),
                         "cores": 1},
            "cpu_model": _cpu_model(),
            "sample": f"{done} tokens in {rows}-token slices of the {wl.n_tok}x{wl.d_in} workload on {n} worker "
                      f"processes (one per core), {dt:.1f} s; one core: {done1} tokens in {dt1:.1f} s; "
                      f"bytes scaled per token"}


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args):
    """--impl reference: the float64 CPU oracle on every host core, rank 0 only.  Each
    step is one bounded sample: a row slice per core, run by one worker process each."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from workloads import make_inputs, workload
    from oracle import wush_oracle as O
    wl = workload(WORKLOAD)
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, wl.G)
    T32 = b["T_wush32"]
    n = host_cores()
    total = max(1, args.steps + args.warmup)
    # about 0.22 ms of one core per token: keep the whole run near a minute or less
    rows = max(1, min(256, int(60.0 / (total * 2.5e-4))))
    per_tok = algorithmic_bytes(wl.n_tok, wl.d_in, wl.G) / wl.n_tok
    with oracle_pool(n) as pool:
        def step(k):
            return sum(pool.map(_oracle_slice, [(x, T32, wl.G, wl.fmt) for x in _slices(inp.x_bits, rows, k * n, n)]))
        step(0)
        for i in range(args.warmup):
            step(i)
        toks, t0 = 0, time.perf_counter()
        for i in range(args.steps):
            toks += step(i)
        dt = time.perf_counter() - t0
    value = toks / dt * per_tok / 1e9
    sample = (f"{rows} tokens per core per step ({n} worker processes, one per core) of the "
              f"{wl.n_tok}x{wl.d_in} workload; bytes scaled per token")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "tokens_per_s": round(toks / dt, 1),
            "config": {"workload": WORKLOAD, "tokens": wl.n_tok, "d_in": wl.d_in, "G": wl.G, "fmt": wl.fmt},
            "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": n, "kind": "oracle",
                             "cpu_model": _cpu_model(), "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _time_calls(fn, stream, n_calls: int, reps: int = 3) -> float:
    """Seconds per call of fn, from CUDA graphs of n_calls launches replayed on stream
    (CUDA events on that stream, best of reps)."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(3):
            fn(i)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_calls):
                fn(i)
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
            best = min(best, e0.elapsed_time(e1) / 1e3 / n_calls)
    del g
    return best


def config_rows(dev, peak_gbs: float) -> dict:
    """The other configurations of the hot path, each timed the same way (graphs, inputs
    rotated over two sets whose total exceeds L2 where the size allows), with its
    algorithmic bytes and fraction of the HBM peak; plus the MXFP4 and NVFP4 GEMM consumers
    at one of the pages' M = 1024 shapes against the FP4 tensor roofline."""
    import numpy as np
    import torch
    import blockwise_adaptive_transforms_b200 as W
    from workloads import make_inputs, workload
    from workloads.synthetic import INT4_SWEEP_TOKENS

    rows = {}
    stream = torch.cuda.Stream(device=dev)

    def bf16_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    def row(name, seconds, nbytes, note=None, **extra):
        r = {"us": round(seconds * 1e6, 3), "GB/s": round(nbytes / seconds / 1e9, 1),
             "hbm_frac": round(nbytes / seconds / 1e9 / peak_gbs, 4), "algorithmic_bytes": nbytes}
        if note:
            r["note"] = note
        r.update(extra)
        rows[name] = r

    # NVFP4 MLP down-projection input, 4096 x 14336, G = 16 (two passes + tensor-scale finalise)
    wl = workload("mlp_down_nvfp4_14336")
    inp = make_inputs(wl)
    T, _ = W.wush_build_transforms(torch.from_numpy(inp.w).to(dev), bf16_dev(inp.xcal_bits), wl.G)
    xs = [bf16_dev(inp.x_bits) for _ in range(2)]
    outs = [W.wush_quant_act(xs[0], T, wl.G, "nvfp4") for _ in range(2)]
    sec = _time_calls(lambda i: W.wush_quant_act(xs[i % 2], T, wl.G, "nvfp4", codes=outs[i % 2][0],
                                                 scales=outs[i % 2][1], tensor_scale=outs[i % 2][2], stream=stream),
                      stream, 20)
    n, d, C = wl.n_tok, wl.d_in, wl.d_in // wl.G
    one_read = n * d * 2 + n * d // 2 + n * C + C * wl.G * wl.G * 4 + 4
    moved = one_read + n * d * 2 + C * wl.G * wl.G * 4
    row("nvfp4_4096x14336", sec, one_read, f"four launches; bytes count X once; the two passes move {moved} B",
        moved_GB_s=round(moved / sec / 1e9, 1))
    # the same call in one cooperative launch (caller workspace): bit-identical outputs
    ws = W.nvfp4_workspace(device=dev, stream=stream)
    sec = _time_calls(lambda i: W.wush_quant_act_nvfp4_onepass(xs[i % 2], T, ws, codes=outs[i % 2][0],
                                                               scales=outs[i % 2][1], tensor_scale=outs[i % 2][2],
                                                               stream=stream), stream, 20)
    row("nvfp4_4096x14336_one_launch", sec, one_read, "wush_quant_act_nvfp4_onepass; bytes count X once",
        moved_GB_s=round(moved / sec / 1e9, 1))
    del xs, outs, inp, ws

    # 70B-like large batch: activations 16384 x 8192 and weights 8192 x 8192, MXFP4
    wl = workload("large_mxfp4_8192")
    inp = make_inputs(wl)
    w_dev = torch.from_numpy(inp.w).to(dev)
    T_act, T_wt = W.wush_build_transforms(w_dev, bf16_dev(inp.xcal_bits), wl.G)   # T_wush, T_xvsh
    n, d, C = wl.n_tok, wl.d_in, wl.d_in // wl.G
    xs = [bf16_dev(inp.x_bits) for _ in range(2)]
    outs = [W.wush_quant_act(xs[0], T_act, wl.G, "mxfp4") for _ in range(2)]
    sec = _time_calls(lambda i: W.wush_quant_act(xs[i % 2], T_act, wl.G, "mxfp4", codes=outs[i % 2][0],
                                                 scales=outs[i % 2][1], stream=stream), stream, 20)
    row("mxfp4_act_16384x8192", sec, algorithmic_bytes(n, d, wl.G))
    del xs, outs
    ws = [w_dev, w_dev.clone()]
    d_out = ws[0].shape[0]
    wouts = [W.wush_quant_weight(ws[0], T_wt, wl.G, "mxfp4") for _ in range(2)]
    sec = _time_calls(lambda i: W.wush_quant_weight(ws[i % 2], T_wt, wl.G, "mxfp4", codes=wouts[i % 2][0],
                                                    scales=wouts[i % 2][1], stream=stream), stream, 20)
    row("mxfp4_weight_8192x8192", sec, d_out * d * 4 + d_out * d // 2 + d_out * C + C * wl.G * wl.G * 4)
    del ws, wouts, inp, w_dev

    # INT4, G = 32, d_in = 4096, token sweep (the small batches are launch-bound)
    wl = workload("int4_sweep_4096")
    inp = make_inputs(wl)
    T, _ = W.wush_build_transforms(torch.from_numpy(inp.w).to(dev), bf16_dev(inp.xcal_bits), wl.G)
    sweep = {}
    for n in INT4_SWEEP_TOKENS:
        xs = [bf16_dev(inp.x_bits[:n]) for _ in range(2)]
        outs = [W.wush_quant_act(xs[0], T, wl.G, "int4") for _ in range(2)]
        sec = _time_calls(lambda i: W.wush_quant_act(xs[i % 2], T, wl.G, "int4", codes=outs[i % 2][0],
                                                     scales=outs[i % 2][1], stream=stream), stream, 50)
        nbytes = n * wl.d_in * 2 + n * wl.d_in // 2 + n * (wl.d_in // wl.G) * 4 + (wl.d_in // wl.G) * wl.G * wl.G * 4
        sweep[str(n)] = {"us": round(sec * 1e6, 3), "GB/s": round(nbytes / sec / 1e9, 1)}
    rows["int4_4096_token_sweep"] = dict(sweep, note="inputs of 1 to 1024 tokens stay in L2; n <= 128 is launch-bound")
    del inp

    # MXFP4 GEMM consumer, M = 1024, N = K = 4096 (Qwen3-8B square projection)
    M, N, K = 1024, 4096, 4096
    g = torch.Generator().manual_seed(7)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(dev)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(dev)
    Tg = (torch.eye(32) + 0.1 * torch.randn(K // 32, 32, 32, generator=g)).to(dev)
    cw, aw = W.wush_quant_weight_mx_atoms(w, Tg)
    cx, ax = W.wush_quant_act_mx_atoms(x, Tg)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    sec = _time_calls(lambda i: W.wush_gemm_mxfp4(cx, ax, cw, aw, out=out, stream=stream), stream, 50)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16_peak, kind = float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        bf16_peak, kind = 1590.0, "fallback"
    tflops = 2.0 * M * N * K / sec / 1e12
    rows["fp4_gemm_1024x4096x4096"] = {"us": round(sec * 1e6, 3), "TFLOP/s": round(tflops, 1),
                                       "tensor_frac": round(tflops / (4 * bf16_peak), 4),
                                       "peak_TFLOP_s": round(4 * bf16_peak, 1),
                                       "peak_source": f"4 x {kind} bf16 (nominal fp4/bf16 ratio)"}
    # the same shape with NVFP4 operands (G = 16 transforms, E4M3 scales, tensor scales)
    Tn = (torch.eye(16) + 0.1 * torch.randn(K // 16, 16, 16, generator=g)).to(dev)
    cwn, awn, twn = W.wush_quant_weight_nv_atoms(w, Tn)
    cxn, axn, txn = W.wush_quant_act_nv_atoms(x, Tn)
    sec = _time_calls(lambda i: W.wush_gemm_nvfp4(cxn, axn, txn, cwn, awn, twn, out=out, stream=stream), stream, 50)
    tflops = 2.0 * M * N * K / sec / 1e12
    rows["nvfp4_gemm_1024x4096x4096"] = {"us": round(sec * 1e6, 3), "TFLOP/s": round(tflops, 1),
                                         "tensor_frac": round(tflops / (4 * bf16_peak), 4),
                                         "peak_TFLOP_s": round(4 * bf16_peak, 1),
                                         "peak_source": f"4 x {kind} bf16 (nominal fp4/bf16 ratio)"}
    torch.cuda.synchronize()
    return rows


def run_native(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    import blockwise_adaptive_transforms_b200 as W
    from workloads import make_inputs, workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = workload(WORKLOAD)
    inp = make_inputs(wl)
    G, n, d = wl.G, wl.n_tok, wl.d_in
    C = d // G
    step_bytes = algorithmic_bytes(n, d, G)

    # transforms: built on the device from the weights and calibration activations
    w_dev = torch.from_numpy(inp.w).to(dev)
    xcal_dev = torch.from_numpy(inp.xcal_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    tb0 = time.perf_counter()
    T, _ = W.wush_build_transforms(w_dev, xcal_dev, G)
    torch.cuda.synchronize()
    build_ms = (time.perf_counter() - tb0) * 1e3
    del w_dev, xcal_dev

    x_host = torch.from_numpy(inp.x_bits.view(np.int16)).view(torch.bfloat16)
    xs = [x_host.to(dev) for _ in range(N_SETS)]
    codes = [torch.empty((n, d // 2), dtype=torch.uint8, device=dev) for _ in range(N_SETS)]
    scales = [torch.empty((n, C), dtype=torch.uint8, device=dev) for _ in range(N_SETS)]
    stream = torch.cuda.Stream(device=dev)

    def launch(i):
        k = i % N_SETS
        W.wush_quant_act(xs[k], T, G, wl.fmt, codes=codes[k], scales=scales[k], stream=stream)

    span_launches = -(-max(args.steps, args.span_launches) // GRAPH_LEN) * GRAPH_LEN

    def capture(fn):
        """Warm-up launches, then one graph of GRAPH_LEN launches, replayed once (its first
        replay uploads it to the device)."""
        with torch.cuda.stream(stream):
            for i in range(min(max(args.warmup, 3), 64)):
                fn(i)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(GRAPH_LEN):
                    fn(i)
            done = min(max(args.warmup, 3), 64)
            while done < args.warmup:
                g.replay()
                done += GRAPH_LEN
            g.replay()
            stream.synchronize()
        return g

    def timed_spans(g):
        """N_SPANS spans of span_launches launches each, every span bracketed by a barrier
        + synchronize and events on the launching stream; seconds per span, max over ranks."""
        out = []
        for _ in range(N_SPANS):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                t0.record(stream)
                for _ in range(span_launches // GRAPH_LEN):
                    g.replay()
                t1.record(stream)
            t1.synchronize()
            out.append(max_over_ranks(t0.elapsed_time(t1) / 1e3, dev))
        return out

    graph = capture(launch)
    st, bits = W.wush_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} after warm-up")
    with ClockSampler(local) as clocks:
        spans = timed_spans(graph)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st, bits = W.wush_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} after the timed region")
    del graph
    span_s = statistics.median(spans)
    per_launch_s = span_s / span_launches
    elapsed_s = per_launch_s * args.steps          # K steps at the median span's rate
    value = job_throughput(world, span_launches, step_bytes, span_s)

    # H+Quant comparator: the same kernel with one shared G x G Hadamard matrix (written
    # by the library), same inputs, outputs, launch count and timing method (the pages
    # compare the two fused kernels)
    H = W.wush_hadamard(G, device=dev)

    def launch_h(i):
        k = i % N_SETS
        W.wush_quant_act_shared(xs[k], H, G, wl.fmt, codes=codes[k], scales=scales[k], stream=stream)

    graph_h = capture(launch_h)
    h_spans = timed_spans(graph_h)
    del graph_h
    h_per_launch_s = statistics.median(h_spans) / span_launches
    h_bytes = step_bytes - C * G * G * 4 + G * G * 4
    st, bits = W.wush_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} after the H+Quant timing")
    tokens_s = world * args.steps * n / elapsed_s
    achieved = step_bytes / per_launch_s / 1e9
    peak, peak_kind = hbm_peak()

    # end to end through the public API: pinned host x -> device, kernel, codes + scales ->
    # pinned host, every step.  Three streams and two buffer sets pipeline the steps: step
    # i's host-to-device copy runs beside step i-1's kernel and step i-2's device-to-host
    # copy (the two copy directions use separate engines); events order each buffer's reuse.
    NB = 2
    x_pin = x_host.pin_memory()
    c_pins = [torch.empty((n, d // 2), dtype=torch.uint8).pin_memory() for _ in range(NB)]
    s_pins = [torch.empty((n, C), dtype=torch.uint8).pin_memory() for _ in range(NB)]
    s_h2d = torch.cuda.Stream(device=dev)
    s_d2h = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(NB)]      # x landed in xs[b]
    ev_run = [torch.cuda.Event() for _ in range(NB)]     # kernel on buffer b done
    ev_out = [torch.cuda.Event() for _ in range(NB)]     # codes/scales of buffer b copied out
    for b in range(NB):                                  # all "done" at the start
        ev_run[b].record(stream)
        ev_out[b].record(stream)

    def e2e_step(i):
        b = i % NB
        s_h2d.wait_event(ev_run[b])                      # the kernel that read xs[b] is done
        with torch.cuda.stream(s_h2d):
            xs[b].copy_(x_pin, non_blocking=True)
        ev_in[b].record(s_h2d)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])                     # codes[b], scales[b] were copied out
        W.wush_quant_act(xs[b], T, G, wl.fmt, codes=codes[b], scales=scales[b], stream=stream)
        ev_run[b].record(stream)
        s_d2h.wait_event(ev_run[b])
        with torch.cuda.stream(s_d2h):
            c_pins[b].copy_(codes[b], non_blocking=True)
            s_pins[b].copy_(scales[b], non_blocking=True)
        ev_out[b].record(s_d2h)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(s_h2d)
    for i in range(args.e2e_steps):
        e2e_step(i)
    f1.record(s_d2h)
    f1.synchronize()
    torch.cuda.synchronize()
    e2e_s = max_over_ranks(f0.elapsed_time(f1) / 1e3, dev)
    e2e_value = job_throughput(world, args.e2e_steps, step_bytes, e2e_s)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, wl, args.cpu_seconds)
    rows = None
    if world == 1 and not args.no_rows:
        del xs, codes, scales
        torch.cuda.empty_cache()
        rows = config_rows(dev, peak)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    clk = clocks.summary()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_launch_s * 1e3, 6),
        "launches_timed": N_SPANS * span_launches,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "tokens_per_s": round(tokens_s, 1),
        "hbm_roofline_frac": round(achieved / peak, 4),
        "config": {"workload": WORKLOAD, "tokens": n, "d_in": d, "G": G, "fmt": wl.fmt,
                   "l2": f"{N_SETS} rotating input/output sets ({N_SETS * step_bytes / 1e6:.0f} MB > 126 MB L2)",
                   "launch": f"CUDA graphs of {GRAPH_LEN} back-to-back launches",
                   "timing": f"median of {N_SPANS} spans of {span_launches} launches each "
                             f"(span times {', '.join(f'{1e6 * t / span_launches:.3f}' for t in spans)} us per launch)",
                   "transform_build_ms": round(build_ms, 2)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": measured_traffic(),
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback", "algorithmic_bytes_per_launch": step_bytes},
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": n * d * 2,
                "d2h_bytes_per_step": n * d // 2 + n * C, "steps": args.e2e_steps,
                "overlap": "each step's copy in, kernel and copy out on three streams, beside its neighbours"},
        "h_quant": {"value": round(world * h_bytes / h_per_launch_s / 1e9, 2),
                    "unit": "GB/s", "us_per_launch": round(h_per_launch_s * 1e6, 3),
                    "launches": N_SPANS * span_launches,
                    "wush_time_over_h_time": round(per_launch_s / h_per_launch_s, 4),
                    "what": "same fused kernel, one shared Hadamard matrix for every block"},
        "rows": rows,
        "gpu_launches": N_SPANS * span_launches,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
