#!/usr/bin/env python
"""Benchmark of the quantized video-DiT self-attention path on B200.

One step = one full-sequence self-attention call over the workload's
(B, H, N, d) = Wan2.1-14B 720p shape (1, 40, 75600, 128) in INT8/FP8 mode:
the quantization prepass (K mean, smoothing, per-block INT8 Q/K, per-channel
FP8 V) followed by the tcgen05 attention kernel, with the inputs resident in
HBM.  Metric: attention TFLOPS = 4 * B * H * N^2 * d / step time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--mode int8_fp8|bf16]
  python bench.py --op linear [--linear-workload NAME]

`--op ulysses` times the sequence-parallel layer instead: each of N ranks holds
N_seq / N tokens of Q, K, V for all heads; the Ulysses exchange (NCCL
all-to-all) gives each the whole sequence for H / N heads, the INT8/FP8 path
runs on them straight from the receive buffers (the prepass reads the
exchange layout, the attention epilogue writes O into the send layout of the
return exchange), and O goes back.  The total problem is fixed (strong scaling);
value = the full layer's attention FLOPs / max-over-ranks time.  On one GPU
the exchange is a single-rank NCCL all-to-all (a local copy).

`--op stack` times the layer-selective stack as one unit: 40 consecutive
attention calls at B=1, H=40, N=32760, d=128 with seed = layer index, the
modes from attn_layer_schedule (layers 0, 8, 16, 24, 32 in BF16, the rest
INT8/FP8, prepass included); one step = the whole stack.  It also times the
same 40 calls all in BF16 for comparison and splits the time by mode.

`--op linear` times the W8A8 linear layer with 128 x 128 block scales
instead (one step = block-quantize the activations X [M, K] + the block-scaled
INT8 GEMM against pre-quantized weights W [N, K], plus bias), at the
Wan2.1-14B 720p projection shape 75600 x 5120 x 5120 by default; metric
TOPS = 2 * M * N * K / step time.  `--linear-mode w8a16` times the W8A16
fallback (dequantize the 8-bit weights + bf16 GEMM), `--linear-mode bf16` the
plain bf16 layer.

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
device (independent attention calls; no data-path collective), so scaling is
weak and value = all ranks' FLOPs / max-over-ranks time.  The inputs (2.3 GB
of bf16 Q/K/V) are far larger than the 126 MB L2, so no explicit flush is
needed between steps.

`--impl reference` times the CPU oracle (plain C, OpenMP) on a bounded sample
of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

DEFAULT_WORKLOAD = "wan14b_720p"
# Attention-kernel DRAM bytes (read + write) per full launch, from ncu captures
# (dram__bytes_read.sum + dram__bytes_write.sum) of the same kernels on 4 heads
# of the same shape, scaled by heads (each head's operands are read from DRAM
# once).  Keyed by (workload, H, mode); absent keys report null.
NCU_TRAFFIC_BYTES = {
    ("wan14b_720p", 40, "int8_fp8"): 1.650e9,
    ("wan14b_720p", 40, "bf16"): 3.006e9,
}
# Linear GEMM DRAM bytes per launch (ncu captures of the same kernels at the
# same shape), keyed by (workload, linear mode).  Absent keys report null.
NCU_TRAFFIC_BYTES_LINEAR = {
    ("wan14b_720p_proj", "w8a8"): 1.152e9,
    ("wan14b_720p_proj", "w8a16"): 3.477e9,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 20 for attention, 400 for --op linear)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--heads", type=int, default=0, help="override H (small profiling captures)")
    ap.add_argument("--mode", default="int8_fp8", choices=["int8_fp8", "bf16", "int8_fp8_qtoken"])
    ap.add_argument("--e2e-steps", type=int, default=3, help="end-to-end steps (at least 1)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=4096)
    ap.add_argument("--op", default="attention", choices=["attention", "linear", "ulysses", "stack"])
    ap.add_argument("--linear-workload", default="wan14b_720p_proj", choices=sorted(synth.LINEAR_WORKLOADS))
    ap.add_argument("--linear-mode", default="w8a8", choices=["w8a8", "w8a16", "bf16"])
    return ap.parse_args()


def workload(args):
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        from dataclasses import replace
        w = replace(w, H=args.heads)
    return w


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank value over all ranks (identity at world size 1)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank: int):
    """Each rank attends over its own batch element: same shape, seed offset by rank."""
    return w.with_seed(w.seed + rank)


# Exponentials per clock per SM: the SFU's ex2 rate (16 results/clk/SM; a microbenchmark with two issuing
# warps per sub-partition measured 3.9 per clock per sub-partition).
SFU_EX2_PER_CLK_PER_SM = 16.0


def sfu_cap_tflops(d: int, sms: int, sm_mhz):
    """The attention FLOP rate one ex2 per score allows: a call does 4*N^2*d FLOPs over N^2 exponentials,
    so 4*d FLOPs per SFU result.  None without a clock reading."""
    if not sm_mhz:
        return None
    return 4.0 * d * SFU_EX2_PER_CLK_PER_SM * sms * float(sm_mhz) * 1e6 / 1e12


def sfu_cap(d: int, sms: int, sm_mhz, achieved: float):
    cap = sfu_cap_tflops(d, sms, sm_mhz)
    return {"tflops": cap, "frac": (achieved / cap) if cap else None,
            "basis": "one ex2 per score at 16 results/clk/SM and the median SM clock"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_baseline(w, n_rows: int, impl_line: bool = False):
    """The oracle as it stands, on a bounded sample: prepass of head 0 plus the
    emulated quantized attention for n_rows sampled query rows of that head."""
    import oracle
    w1 = synth.Workload(w.name, 1, 1, w.N, w.d, seed=w.seed, k_off_std=w.k_off_std,
                        outlier_frac=w.outlier_frac, outlier_scale=w.outlier_scale, zero_k_channel=w.zero_k_channel)
    q, k, v = synth.qkv_numpy(w1)
    rows = synth.sample_rows(w.seed + 7, w.N, n_rows)
    t0 = time.perf_counter()
    pre = oracle.prepass(q, k, v)
    oracle.attn_emul(pre, rows)
    dt = time.perf_counter() - t0
    flops = 4.0 * len(rows) * w.N * w.d
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
            "sample": f"K-mean/INT8/FP8 prepass of 1 head + emulated attention of {len(rows)} sampled query rows "
                      f"of that head (N={w.N}, d={w.d}); TFLOPS = 4*rows*N*d/time",
            "seconds": dt}


def attention_config(w, args, world: int) -> dict:
    """The config of an attention line; the reference arm prints the same one."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "mode": args.mode,
            "global_batch": world * w.B, "parallelism": f"independent calls x{world}",
            "l2": "inputs (2.3 GB) larger than L2; no flush"}


def linear_config(w, world: int) -> dict:
    return {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "global_batch": world,
            "parallelism": f"independent calls x{world}", "l2": "X (774 MB bf16) larger than L2; no flush"}


def stack_config(base, world: int) -> dict:
    return {"workload": "layer_stack", "layers": synth.LAYER_STACK_LAYERS, "B": base.B, "H": base.H, "N": base.N,
            "d": base.d, "full_precision_layers": list(synth.LAYER_STACK_FULL_PRECISION), "seeds": "layer index",
            "parallelism": f"independent stacks x{world}", "l2": "every layer's inputs (1.0 GB) larger than L2; no flush"}


def run_reference_linear(args, rank, world):
    """Reference arm of --op linear: the CPU oracle on a bounded sample per step."""
    w = synth.LINEAR_WORKLOADS[args.linear_workload]
    if rank != 0:
        return
    vals, secs = [], []
    for i in range(max(args.warmup, 0) + args.steps):
        r = cpu_baseline_linear(w, 64 if i < args.warmup else 256)
        if i >= args.warmup:
            vals.append(r["value"])
            secs.append(r["seconds"])
    tops = statistics.median(vals)
    print(json.dumps({
        "impl": "reference", "op": "linear_w8a8", "metric": "W8A8 linear TOPS per call (2*M*N*K)", "value": tops,
        "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int64 block sums, f32 (CPU oracle)", "data": "synthetic",
        "config": linear_config(w, world),
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": r["cores"], "kind": "oracle", "sample": r["sample"]},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle, timed on the host cores, same metric."""
    if args.op == "linear":
        run_reference_linear(args, rank, world)
        return
    # the stack's calls all have the layer-stack shape; one sampled call per step stands for them
    w = synth.WORKLOADS["layer_stack"] if args.op == "stack" else workload(args)
    if rank != 0:
        return
    rows = max(64, args.cpu_rows // 8)
    for _ in range(max(args.warmup, 0)):
        cpu_baseline(w, 64)
    vals, secs = [], []
    for _ in range(args.steps):
        r = cpu_baseline(w, rows)
        vals.append(r["value"])
        secs.append(r["seconds"])
    tflops = statistics.median(vals)
    metric = "attention TFLOPS per call (4*B*H*N^2*d)" + (", 40-layer selective stack" if args.op == "stack" else "")
    line = {
        "impl": "reference", "metric": metric, "value": tflops,
        "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64/f32 (CPU oracle)", "data": "synthetic",
        "config": stack_config(w, world) if args.op == "stack" else attention_config(w, args, world),
        "cpu_baseline": {"value": tflops, "unit": "TFLOPS", "cores": r["cores"], "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": tflops, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from video_dit_quantized_b200 import sage

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload(args)
    mode = {"int8_fp8": sage.MODE_INT8_FP8, "bf16": sage.MODE_BF16, "int8_fp8_qtoken": sage.MODE_INT8_FP8_QTOKEN}[args.mode]
    quant = mode != sage.MODE_BF16
    qgran = 1 if mode == sage.MODE_INT8_FP8_QTOKEN else 128
    wr = rank_workload(w, rank)
    q_h, k_h, v_h = synth.qkv_torch(wr, pin=True)
    q, k, v = (t.to(dev, non_blocking=True) for t in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    ws = sage.alloc_workspace(w.B, w.H, w.N, w.d, mode, dev)
    nT = (w.N + 127) // 128
    pre = None
    if quant:
        pre = dict(
            q_i8=torch.empty((w.B, w.H, nT * 128, w.d), dtype=torch.int8, device=dev),
            q_scale=torch.empty((w.B, w.H, nT * 128 if qgran == 1 else nT), dtype=torch.float32, device=dev),
            k_i8=torch.empty((w.B, w.H, nT * 128, w.d), dtype=torch.int8, device=dev),
            k_scale=torch.empty((w.B, w.H, nT), dtype=torch.float32, device=dev),
            k_mean=torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=dev),
            v_f8t=torch.empty((w.B, w.H, w.d, nT * 128), dtype=torch.uint8, device=dev),
            v_scale=torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=dev),
        )
        scratch = torch.empty(max(sage.prepass_scratch_bytes(w.B, w.H, w.N, w.d), 256), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    sp = sage._stream(stream)
    P = sage._ptr

    def step(ev=None):
        """One pass of the path; ev = (start, after_prepass, end) events or None."""
        if ev:
            ev[0].record(stream)
        if quant:
            rc = sage.LIB.sage_quantize_qk_ex(P(q), P(k), P(v), w.B, w.H, w.N, w.d, qgran, P(pre["q_i8"]),
                                              P(pre["q_scale"]), P(pre["k_i8"]), P(pre["k_scale"]), P(pre["k_mean"]),
                                              P(pre["v_f8t"]), P(pre["v_scale"]), P(scratch), scratch.numel(), sp)
            if rc:
                raise sage.SageError(rc, "sage_quantize_qk_ex")
            if ev:
                ev[1].record(stream)
            rc = sage.LIB.sage_attn_quantized_ex(P(pre["q_i8"]), P(pre["q_scale"]), P(pre["k_i8"]),
                                                 P(pre["k_scale"]), P(pre["v_f8t"]), P(pre["v_scale"]), P(o), w.B, w.H,
                                                 w.N, w.d, qgran, P(ws), sp)
            if rc:
                raise sage.SageError(rc, "sage_attn_quantized_ex")
        else:
            if ev:
                ev[1].record(stream)
            rc = sage.LIB.sage_attn_fwd(P(q), P(k), P(v), P(o), w.B, w.H, w.N, w.d, mode, P(ws), ws.numel(), sp)
            if rc:
                raise sage.SageError(rc, "sage_attn_fwd")
        if ev:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = sage.status(ws)
    if st != sage.OK:
        raise sage.SageError(st, "warm-up")

    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = t_start.elapsed_time(t_end)
    prep_ms = [a.elapsed_time(b) for a, b, _ in evs]
    attn_ms = [b.elapsed_time(c) for _, b, c in evs]
    step_ms = [a.elapsed_time(c) for a, _, c in evs]
    st = sage.status(ws)
    if st != sage.OK:
        raise sage.SageError(st, "timed region")

    total_ms = max_over_ranks(total_ms, world, dev)

    # ---- end to end: pinned host inputs -> public host-buffer call -> host output ----
    # sage_attn_fwd_host copies each chunk of heads in, runs the path on it and
    # copies its output out, overlapping the copies of one chunk with the
    # attention of another; every step moves all of Q, K, V in and all of O out.
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    chunk = sage.host_chunk_heads(w.B, w.H, w.N, w.d)
    ws_e2e = sage.alloc_host_workspace(w.B, w.H, w.N, w.d, mode, chunk, dev)
    staging = tuple(torch.empty_like(q) for _ in range(4))
    h2d = 3 * q.numel() * q.element_size()
    d2h = o.numel() * o.element_size()

    def e2e_step():
        sage.attn_fwd_host(q_h, k_h, v_h, o_h, mode, staging=staging, workspace=ws_e2e, chunk_heads=chunk,
                           stream=stream)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / max(args.e2e_steps, 1), world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_rows)
        cpu.pop("seconds", None)
    # the tensor-core rate the kernel is bounded by, measured per SM per clock on this GPU (MMA-only probe)
    probe = sage.dbg_mma_peak(sage.MMA_I8 if quant else sage.MMA_BF16, 256, iters=2000)

    if rank != 0:
        return
    flops = w.flops
    ms_step = total_ms / args.steps
    value = world * flops / (ms_step * 1e-3) / 1e12
    peaks, src = load_peaks()
    # dense contraction peak for the kernel's own dtype: INT8/FP8 = 2x the measured
    # bf16 figure (nominal 4.5 vs 2.25 PFLOP/s); the sustained figure, since the
    # kernel runs back to back for seconds under the power cap.
    ratio = 2.0 if quant else 1.0
    peak = ratio * float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    attn_avg = statistics.mean(attn_ms)
    achieved = flops / (attn_avg * 1e-3) / 1e12
    clocks = clk.summary()
    traffic = NCU_TRAFFIC_BYTES.get((w.name, w.H, args.mode))
    line = {
        "metric": "attention TFLOPS per call (4*B*H*N^2*d)",
        "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8/fp8e4m3 (fp32 accumulate)" if quant else "bf16 (fp32 accumulate)",
        "data": "synthetic",
        "config": attention_config(w, args, world),
        "kernels_ms": {"prepass_median": statistics.median(prep_ms), "attention_median": statistics.median(attn_ms),
                       "attention_p10": float(np.percentile(attn_ms, 10)),
                       "attention_p90": float(np.percentile(attn_ms, 90)),
                       "attention_min": min(attn_ms), "attention_max": max(attn_ms),
                       "step_p10": float(np.percentile(step_ms, 10)), "step_p90": float(np.percentile(step_ms, 90))},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_basis": f"{'2x ' if ratio == 2 else ''}bf16_tflops_sustained ({src})",
                     "frac_of_datasheet_4500": achieved / (4500.0 if ratio == 2 else 2250.0),
                     "sfu_cap": sfu_cap(w.d, probe["sms"], clocks["sm_mhz"], achieved)},
        "cpu_baseline": cpu,
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        # prepass (statistics, finalize, quantize) + attention; BF16: attention only
        "gpu_launches": args.steps * (4 if quant else 1),
        "mma_probe": {"kind": "i8" if quant else "bf16", "mac_per_clk_per_sm": probe["mac_per_clk_per_sm"],
                      "peak_at_median_sm_clock_tflops": (2 * probe["mac_per_clk_per_sm"] * probe["sms"] *
                                                         (clocks["sm_mhz"] or 0) * 1e6 / 1e12),
                      "frac_of_it": (achieved / (2 * probe["mac_per_clk_per_sm"] * probe["sms"] *
                                                 clocks["sm_mhz"] * 1e6 / 1e12)) if clocks["sm_mhz"] else None},
        "e2e_api": f"sage_attn_fwd_host (pinned host Q/K/V in, O out, pipelined over chunks of {chunk} heads)",
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_linear(w, n_rows: int):
    """The oracle as it stands on a bounded sample: 2-D block quantization of the
    128-row blocks holding n_rows sampled rows of X, and the block-scaled GEMM
    of those rows against the (pre-quantized) weights."""
    import oracle
    x, wt, b = synth.linear_numpy(w)
    wq, sw = oracle.quant_blocks_2d(wt)
    rows = synth.sample_rows(w.seed + 7, w.M, n_rows)
    blocks = np.unique(rows // 128)
    t0 = time.perf_counter()
    xs = np.concatenate([x[r * 128:(r + 1) * 128] for r in blocks])
    xq, sx = oracle.quant_blocks_2d(xs)
    local = np.array([np.searchsorted(blocks, r // 128) * 128 + r % 128 for r in rows], dtype=np.int32)
    oracle.linear_w8a8(xq, sx, wq, sw, b, local)
    dt = time.perf_counter() - t0
    ops = 2.0 * len(rows) * w.N * w.K
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle",
            "sample": f"128x128 block quantization of the {len(blocks)} row blocks holding {len(rows)} sampled rows "
                      f"of X + block-scaled INT8 GEMM of those rows (N={w.N}, K={w.K}); TOPS = 2*rows*N*K/time",
            "seconds": dt}


def run_linear(args, rank, world, local_rank):
    """W8A8 linear: block-quantize X, block-scaled INT8 GEMM (+ bias) against pre-quantized W."""
    import torch
    import torch.distributed as dist
    from video_dit_quantized_b200 import sage

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.LINEAR_WORKLOADS[args.linear_workload]
    wr = w if rank == 0 else synth.LinearWorkload(w.name, w.M, w.N, w.K, seed=w.seed + rank,
                                                  outlier_frac=w.outlier_frac, outlier_scale=w.outlier_scale)
    x_np, w_np, b_np = synth.linear_numpy(wr)
    as_bf16 = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    x_h = as_bf16(x_np).pin_memory()
    x = x_h.to(dev)
    wt, bias = as_bf16(w_np).to(dev), as_bf16(b_np).to(dev)
    stream = torch.cuda.current_stream()
    nk = w.K // 128
    wq, sw = sage.quantize_blocks_2d(wt)                  # weights: quantized once, outside the step
    lmode = args.linear_mode
    ws16 = torch.empty(int(sage.LIB.sage_linear_w8a16_workspace_bytes(w.N, w.K)), dtype=torch.uint8, device=dev)
    xq = torch.empty((w.M, w.K), dtype=torch.int8, device=dev)
    sx = torch.empty(((w.M + 127) // 128, nk), dtype=torch.float32, device=dev)
    y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(64, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    sp = sage._stream(stream)
    P = sage._ptr

    def step(ev=None):
        """w8a8: quantize X | GEMM; w8a16: dequantize W | bf16 GEMM; bf16: - | bf16 GEMM."""
        if ev:
            ev[0].record(stream)
        if lmode == "w8a8":
            rc = sage.LIB.sage_quantize_blocks_2d(P(x), w.M, w.K, P(xq), P(sx), sp)
        elif lmode == "w8a16":
            rc = sage.LIB.sage_dequant_blocks_2d(P(wq), P(sw), w.N, w.K, P(ws16), sp)
        else:
            rc = 0
        if rc:
            raise sage.SageError(rc, "quantize / dequantize")
        if ev:
            ev[1].record(stream)
        if lmode == "w8a8":
            rc = sage.LIB.sage_linear_w8a8(P(xq), P(sx), P(wq), P(sw), P(bias), P(y), sage.DTYPE_BF16, w.M, w.N, w.K,
                                           P(status), sp)
        else:
            rc = sage.LIB.sage_linear_bf16(P(x), P(ws16 if lmode == "w8a16" else wt), P(bias), P(y), sage.DTYPE_BF16,
                                           w.M, w.N, w.K, P(status), sp)
        if rc:
            raise sage.SageError(rc, "linear")
        if ev:
            ev[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sage.status(status) != sage.OK:
        raise sage.SageError(sage.ETIMEOUT, "warm-up")
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    quant_ms = [a.elapsed_time(b) for a, b, _ in evs]
    gemm_ms = [b.elapsed_time(c) for _, b, c in evs]
    if sage.status(status) != sage.OK:
        raise sage.SageError(sage.ETIMEOUT, "timed region")

    # end to end through the binding: pinned host X in, bf16 Y out, every step
    y_h = torch.empty((w.M, w.N), dtype=torch.bfloat16, pin_memory=True)

    def e2e_step():
        x.copy_(x_h, non_blocking=True)
        if lmode == "w8a8":
            sage.quantize_blocks_2d(x, xq, sx, stream=stream)
            sage.linear_w8a8(xq, sx, wq, sw, bias, y=y, status=status, stream=stream)
        elif lmode == "w8a16":
            sage.linear_w8a16(x, wq, sw, bias, y=y, workspace=ws16, status=status, stream=stream)
        else:
            sage.linear_bf16(x, wt, bias, y=y, status=status, stream=stream)
        y_h.copy_(y, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / max(args.e2e_steps, 1), world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and lmode == "w8a8":
        cpu = cpu_baseline_linear(w, 1024)
        cpu.pop("seconds", None)
    if rank != 0:
        return
    ms_step = total_ms / args.steps
    peaks, src = load_peaks()
    ratio = 2.0 if lmode == "w8a8" else 1.0
    peak = ratio * float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    gemm_avg = statistics.mean(gemm_ms)
    achieved = w.flops / (gemm_avg * 1e-3) / 1e12
    line = {
        "op": f"linear_{lmode}",
        "metric": f"{lmode.upper()} linear TOPS per call (2*M*N*K)",
        "value": world * w.flops / (ms_step * 1e-3) / 1e12, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8 (int32 block sums, fp32 accumulate)" if lmode == "w8a8" else "bf16 (fp32 accumulate)",
        "data": "synthetic",
        "config": linear_config(w, world),
        "kernels_ms": {("quantize_median" if lmode == "w8a8" else "dequantize_median"): statistics.median(quant_ms),
                       "gemm_median": statistics.median(gemm_ms),
                       "gemm_min": min(gemm_ms), "gemm_max": max(gemm_ms)},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": NCU_TRAFFIC_BYTES_LINEAR.get((w.name, lmode)),
                     "peak_basis": f"{'2x ' if ratio == 2 else ''}bf16_tflops_sustained ({src})",
                     "frac_of_datasheet": achieved / (4500.0 if ratio == 2 else 2250.0)},
        "cpu_baseline": cpu,
        "e2e": {"value": world * w.flops / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS",
                "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": y.numel() * 2, "ms_per_step": e2e_ms},
        "gpu_launches": (1 if lmode == "bf16" else 2) * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_ulysses(args, rank, world, local_rank):
    """Sequence-parallel attention layer: Ulysses exchange around the INT8/FP8 path."""
    import torch
    import torch.distributed as dist
    from video_dit_quantized_b200 import sage
    from video_dit_quantized_b200.ulysses import UlyssesAttention

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload(args)
    if w.N % world or w.H % world:
        raise SystemExit(f"N={w.N} and H={w.H} must be divisible by the {world} ranks")
    Nl = w.N // world
    mode = {"int8_fp8": sage.MODE_INT8_FP8, "bf16": sage.MODE_BF16, "int8_fp8_qtoken": sage.MODE_INT8_FP8_QTOKEN}[args.mode]
    full = synth.qkv_torch(w)                                   # the same seeded layer on every rank
    mine = [t.permute(0, 2, 1, 3)[:, rank * Nl:(rank + 1) * Nl].contiguous().to(dev) for t in full]
    del full
    ua = UlyssesAttention(w.B, Nl, w.H, w.d, world, mode=mode, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        return ua(*mine)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sage.status(ua.workspace) != sage.OK:
        raise sage.SageError(sage.ETIMEOUT, "warm-up")
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    if sage.status(ua.workspace) != sage.OK:
        raise sage.SageError(sage.ETIMEOUT, "timed region")
    if rank != 0:
        return
    print(json.dumps({
        "op": "ulysses_attention",
        "metric": "attention TFLOPS per call (4*B*H*N^2*d), sequence-parallel layer",
        "value": w.flops / (ms * 1e-3) / 1e12, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "int8/fp8e4m3 (fp32 accumulate)" if mode != sage.MODE_BF16 else "bf16 (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "mode": args.mode,
                   "parallelism": f"ulysses sp{world}", "tokens_per_rank": Nl, "heads_per_rank": w.H // world},
        # send copies of q, k, v and the O receive copy (none at P = 1: the layouts coincide), then the
        # prepass (three kernels) + attention (BF16: three gathers + attention)
        "gpu_launches": args.steps * ((4 if world > 1 else 0) + 4),
        "clocks": clk.summary(),
    }), flush=True)


def run_stack(args, rank, world, local_rank):
    """The 40-call layer-selective stack (one step = all 40 calls, each with its own seeded inputs)."""
    import torch
    import torch.distributed as dist
    from video_dit_quantized_b200 import sage

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base = synth.WORKLOADS["layer_stack"]
    L = synth.LAYER_STACK_LAYERS
    modes = sage.layer_schedule(L, synth.LAYER_STACK_FULL_PRECISION)
    host, inputs = [], []
    for layer in range(L):
        # every rank runs its own independent stack: layer seeds offset by rank
        h = synth.qkv_torch(base.with_seed(layer + rank * L), pin=True)
        host.append(h)
        inputs.append(tuple(t.to(dev, non_blocking=True) for t in h))
    o = torch.empty_like(inputs[0][0])
    ws = sage.alloc_workspace(base.B, base.H, base.N, base.d, sage.MODE_INT8_FP8, dev)
    stream = torch.cuda.current_stream()
    sp = sage._stream(stream)
    P = sage._ptr
    torch.cuda.synchronize()

    def stack(layer_modes, evs=None):
        for layer in range(L):
            q, k, v = inputs[layer]
            if evs:
                evs[layer][0].record(stream)
            rc = sage.LIB.sage_attn_fwd(P(q), P(k), P(v), P(o), base.B, base.H, base.N, base.d, layer_modes[layer],
                                        P(ws), ws.numel(), sp)
            if rc:
                raise sage.SageError(rc, "sage_attn_fwd")
            if evs:
                evs[layer][1].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(layer_modes):
        for _ in range(args.warmup):
            stack(layer_modes)
        torch.cuda.synchronize()
        evs = [[tuple(torch.cuda.Event(enable_timing=True) for _ in range(2)) for _ in range(L)]
               for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clk:
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for i in range(args.steps):
                stack(layer_modes, evs[i])
            t1.record(stream)
            torch.cuda.synchronize()
            barrier()
        st = sage.status(ws)
        if st != sage.OK:
            raise sage.SageError(st, "stack")
        per_call = [[a.elapsed_time(b) for a, b in step] for step in evs]
        return max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps, per_call, clk.summary()

    ms, per_call, clocks = timed(modes)
    ms_bf16, _, clocks_bf16 = timed([sage.MODE_BF16] * L)

    # end to end: every layer's Q, K, V from pinned host memory through the public host-buffer call,
    # its O back to pinned host memory
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    chunk = sage.host_chunk_heads(base.B, base.H, base.N, base.d)
    ws_e2e = sage.alloc_host_workspace(base.B, base.H, base.N, base.d, sage.MODE_INT8_FP8, chunk, dev)
    staging = tuple(torch.empty_like(o) for _ in range(4))

    def e2e_stack():
        for layer in range(L):
            sage.attn_fwd_host(*host[layer], o_h, modes[layer], staging=staging, workspace=ws_e2e,
                               chunk_heads=chunk, stream=stream)

    e2e_stack()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_stack()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if rank != 0:
        return
    flops = L * base.flops
    peaks, src = load_peaks()
    sustained = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    by_mode = {}
    for name, m, pk in (("int8_fp8", sage.MODE_INT8_FP8, 2.0 * sustained), ("bf16", sage.MODE_BF16, sustained)):
        calls = [c for step in per_call for c, mm in zip(step, modes) if mm == m]
        avg = statistics.mean(calls)
        ach = base.flops / (avg * 1e-3) / 1e12
        by_mode[name] = {"calls_per_stack": sum(1 for mm in modes if mm == m), "ms_per_call_mean": avg,
                         "achieved": ach, "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
                         "peak_basis": f"{'2x ' if m != sage.MODE_BF16 else ''}bf16_tflops_sustained ({src})"}
    h2d = L * 3 * o.numel() * o.element_size()
    d2h = L * o.numel() * o.element_size()
    print(json.dumps({
        "op": "layer_stack",
        "metric": "attention TFLOPS per call (4*B*H*N^2*d), 40-layer selective stack",
        "value": world * flops / (ms * 1e-3) / 1e12, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8/fp8e4m3 + bf16 layers (fp32 accumulate)", "data": "synthetic",
        "config": stack_config(base, world),
        "by_mode": by_mode,
        "all_bf16_stack": {"ms_per_step": ms_bf16, "tflops": flops / (ms_bf16 * 1e-3) / 1e12,
                           "speedup_of_selective": ms_bf16 / ms, "clocks": clocks_bf16},
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * sum(4 if m != sage.MODE_BF16 else 1 for m in modes),
        "clocks": clocks,
    }), flush=True)


def main():
    args = parse()
    if args.steps is None:
        # a linear step is ~2.5 ms: 400 steps keep the timed region (and its clock samples) near a second
        args.steps = {"linear": 400, "stack": 3}.get(args.op, 20)
    args.e2e_steps = max(1, args.e2e_steps)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1 or args.op == "ulysses":
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(29500 + os.getpid() % 1000))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.op == "ulysses":
            run_ulysses(args, rank, world, local_rank)
        elif args.op == "stack":
            run_stack(args, rank, world, local_rank)
        elif args.op == "linear":
            run_linear(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1 or args.op == "ulysses":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
