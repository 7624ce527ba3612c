#!/usr/bin/env python
"""Benchmark of the DiT block hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --measure-int8-peak      # writes profiles/int8_peak.json
    python bench.py --kernel-sweep           # memory-bound kernels alone, GB/s

One step = one pass of the hot path over one batch of synthetic input.  The
default workload is the 8-block bf16 stack at the 33B-class width: d = 5120
(40 heads x 128, MLP 20480, fp32 residual stream) over 6x32x32 video + 384
audio tokens (S = 6528); one step is one h3b_stack_forward (RoPE table, then
per block RMSNorm, QKV GEMM + RoPE, flash attention, O-proj + residual,
RMSNorm, FC1 + GELU, FC2 + residual).  The same run also times the INT8 W8A8
d = 5120 block over 5x48x84 video + 480 audio tokens (S = 20640) with the same
protocol and reports it as the "int8" sub-record.  Other workloads: the
single d = 3072 block, the 45-block 20-step denoising loop with reuse 2 and
token reduction, the preview loop.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize() on both sides, CUDA events on the launching stream,
max over ranks.  The working set (weights + activations + workspace) exceeds
the 126 MB L2, so no flush is inserted between steps.  N > 1 runs N
independent replicas (one per GPU, launched by torchrun); the path has no
exchange step, so there is no data-path collective ("scaling": "weak").
A second pass of the same K steps records library-owned CUDA events around
every launch for the per-kernel shares and the roofline of the dominant
kernel ("ms_per_step_traced"; the events between launches forgo the overlap
of neighbouring kernels, so `value` comes from the untraced pass).  Tensor
peaks follow the SM clock sampled during the timed region (tensor_peak);
fractions against the datasheet peaks are printed beside them.

--impl reference times the CPU oracle (numpy fp64) on the host cores, one
1/8-block token chunk per step (rank 0 only under torchrun).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "stack8_d5120_s6528"
INT8_WORKLOAD = "block_int8_d5120_s20640"
METRIC = "DiT block tokens/s"
# default timed steps per workload: about 1-30 s of device time each
DEFAULT_STEPS = {"block_d256_s288": 2000, "block_d3072_s6400": 300, "stack8_d5120_s6528": 30,
                 "block_int8_d5120_s20640": 60, "loop45_d5120_s6528": 2,
                 "preview40_d5120_s2784": 4}
# used only when MEASURED_PEAKS.json is absent: an earlier measurement on B200s of
# this kind (copy bandwidth; cuBLAS bf16 burst, and sustained under the 1 kW cap
# at about 1.3 GHz)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "clocks_under_load": {"sm_mhz_median": 1300.0}, "source": "fallback"}
# B200 datasheet dense peaks (bf16, int8) and the HBM figure the block is held to
NOMINAL = {"bf16_tflops": 2250.0, "int8_tops": 4500.0, "hbm_gbs": 8000.0}
INT8_PEAK_FILE = os.path.join(ROOT, "profiles", "int8_peak.json")


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(pk, clocks, int8=False):
    """Dense tensor peak for a kernel timed at the sampled SM clock.

    Two measured points bound it: the burst figure (best single GEMM, high
    clock) and the sustained figure (a seconds-long GEMM loop under the power
    cap, at the median clock recorded with it).  The peak is the sustained
    figure scaled by (median SM clock of this run / that clock), clamped to
    [sustained, burst]: a run at full clock gets the burst peak, one at the
    power-capped clock the sustained peak.  INT8 uses its own measured pair
    when profiles/int8_peak.json exists, else the bf16 pair x 2 (the nominal
    4.5 / 2.25 ratio)."""
    src = ("fallback peaks (no MEASURED_PEAKS.json)" if pk.get("source") == "fallback"
           else "MEASURED_PEAKS.json (cuBLAS bf16)")
    burst, sust = pk.get("bf16_tflops"), pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    f_s = (pk.get("clocks_under_load") or {}).get("sm_mhz_median")
    scale, nominal = 1.0, NOMINAL["bf16_tflops"]
    if int8:
        nominal = NOMINAL["int8_tops"]
        if os.path.exists(INT8_PEAK_FILE):
            q = json.load(open(INT8_PEAK_FILE))
            burst, sust, f_s = q["int8_tops"], q["int8_tops_sustained"], q.get("sustained_sm_mhz_median")
            src = "profiles/int8_peak.json (torch._int_mm int8)"
        else:
            scale = 2.0
            src += " x 2 (nominal int8/bf16 ratio)"
    burst, sust = burst * scale, sust * scale
    med = (clocks or {}).get("sm_mhz")
    if med and f_s:
        peak = min(burst, max(sust, sust * med / f_s))
        basis = (f"{src}: sustained {sust:.0f} x median {med:.0f} MHz / {f_s:.0f} MHz, clamped to "
                 f"[sustained {sust:.0f}, burst {burst:.0f}]")
    else:
        peak = sust
        basis = f"{src}: sustained {sust:.0f} (no clock samples)"
    return {"peak": round(peak, 1), "basis": basis, "nominal": nominal}


def max_over_ranks(ms: float, device) -> float:
    """Slowest rank's time (the job's time) when a process group is up."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_step: float, steps: int, world: int, ms: float) -> float:
    """Units all replicas processed per second of the slowest replica's time."""
    return units_per_step * steps * world / (ms / 1e3)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def src_digest(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "attention": ["audio_diffusion_transformer_dit_b200/csrc/attention.cu",
                  "audio_diffusion_transformer_dit_b200/csrc/common.cuh"],
    "gemm": ["audio_diffusion_transformer_dit_b200/csrc/gemm.cu",
             "audio_diffusion_transformer_dit_b200/csrc/common.cuh"],
    "mem": ["audio_diffusion_transformer_dit_b200/csrc/mem_kernels.cu"],
}


def kernel_family(name):
    if name.startswith("gemm"):
        return "gemm"
    if name == "attention":
        return "attention"
    return "mem"


def measured_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel source (null otherwise)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel}@{workload}")
    if not d:
        return None
    if d.get("src") != src_digest(KERNEL_SOURCES[kernel_family(kernel)]):
        return None
    return d.get("bytes_per_launch")


# ----------------------------------------------------------------------------- per-kernel algorithmic work
def kernel_work(name, wl, dtype, merged=False):
    """(amount, unit, bound) of ONE launch's algorithmic work."""
    S = wl.seq_merged if merged else wl.seq
    d, f = wl.d, wl.ffn
    int8 = dtype == W.INT8
    flops = {"gemm_qkv_rope": 2.0 * S * 3 * d * d, "gemm_o_resid": 2.0 * S * d * d,
             "gemm_fc1_gelu": 2.0 * S * f * d, "gemm_fc2_resid": 2.0 * S * d * f,
             "attention": 4.0 * S * S * d}
    if name in flops:
        unit = "TOP/s" if (int8 and name != "attention") else "TFLOP/s"
        return flops[name], unit, "tensor"
    nbytes = {"rmsnorm": S * d * 4 + S * d * (1 if int8 else 2) + (S * 4 if int8 else 0),
              "quant_rows": S * d * 2 + S * d + S * 4,
              "quant_absmax": S * f * 2 + S * f + S * 8,
              "rope_table": S * (wl.head_dim // 2) * 8,
              "token_merge": wl.seq * d * 4 + wl.seq_merged * d * 4,
              "token_unmerge": wl.seq * d * 4 + wl.seq_merged * d * 4,
              "token_unmerge_delta": 2 * wl.seq * d * 4 + 2 * wl.seq_merged * d * 4,
              "flow_step": wl.seq * d * 4 * 3,
              # folded RMSNorm: each row's partial sums of squares (2 per 256 columns) -> one factor
              "norm_scale": S * (2 * ((d + 255) // 256)) * 4 + S * 4}
    if name in nbytes:
        return float(nbytes[name]), "GB/s", "hbm"
    return None, None, None


# ----------------------------------------------------------------------------- our arm
def build_workload(wl, dev):
    from audio_diffusion_transformer_dit_b200 import h3b
    dm = h3b.dims_of(wl)
    int8 = wl.dtype == W.INT8
    n_layers = wl.n_blocks
    blocks = []
    for layer in range(n_layers):
        w = W.block_weights(wl, layer, dev)
        blocks.append(h3b.Block.quantized(w) if int8 else h3b.Block.from_dict(w))
        del w
    x = W.initial_tokens(wl, dev)
    ws = h3b.workspace(dm, wl.dtype, wl.merge_first >= 0)
    return dm, blocks, x, ws


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def measure(args, wl, dev, world, local):
    """Time K steps of one workload (after W warm-ups) and return its record:
    rate, per-kernel shares from a traced second pass, the dominant kernel's
    roofline, the whole-step roofline and the end-to-end rate through the
    public API with host buffers."""
    from audio_diffusion_transformer_dit_b200 import h3b
    dm, blocks, x, ws = build_workload(wl, dev)
    loop = wl.steps > 0
    v = torch.empty_like(x) if loop else None
    core = loop and args.core_reuse > 0
    n_core = 0

    if loop and (core or args.unmerge_delta or args.cond_rows or args.modulation):
        cond = mod = None
        if args.cond_rows:
            cond = W.normal_tensor((args.cond_rows, wl.d), wl.seed * 7 + 1, dev)
            v = torch.empty((wl.seq + args.cond_rows, wl.d), dtype=torch.float32, device=dev)
        if args.modulation:
            mod = W.normal_tensor((wl.steps, len(blocks), 2, 6, wl.d), wl.seed * 7 + 2, dev, std=0.1)
            mod[..., 2, :] += 1.0
            mod[..., 5, :] += 1.0
        opts = h3b.stack_opts(wl.merge_first, wl.merge_last, args.unmerge_delta,
                              wl.merge_first if core else -1, wl.merge_last if core else -1,
                              cond_rows=cond, modulation=mod)
        ws = h3b.workspace_ex(dm, opts, wl.dtype)
        reuse = 1 if core else wl.reuse

        def step():
            h3b.denoise_ex(dm, blocks, x, v, ws, wl.steps, opts, reuse=reuse,
                           core_reuse=args.core_reuse if core else 1)
        n_fresh = len([i for i in range(wl.steps) if i % reuse == 0 or i == wl.steps - 1])
        n_core = len([i for i in range(wl.steps) if i % args.core_reuse == 0 or i == wl.steps - 1]) if core else 0
        units = 1.0
    elif loop:
        def step():
            h3b.denoise(dm, blocks, x, v, ws, wl.steps, wl.reuse, wl.merge_first, wl.merge_last)
        n_fresh = len([i for i in range(wl.steps) if i % wl.reuse == 0 or i == wl.steps - 1])
        units = 1.0
    elif len(blocks) > 1:
        def step():
            h3b.stack_forward(dm, blocks, x, ws)
        units = float(wl.seq * len(blocks))
    else:
        def step():
            h3b.block_forward(dm, blocks[0], x, ws)
        units = float(wl.seq)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert h3b.device_error() == 0, "device error word set during warm-up"
    eager_step = step
    if args.graph:
        # the whole step captured once; the timed pass replays it (the traced
        # pass below stays eager: replayed launches carry no trace events)
        graph = h3b.Graph(eager_step)
        step = graph.replay
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        assert h3b.device_error() == 0, "device error word set during graph warm-up"

    sampler = ClockSampler(local)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    # Per-kernel durations: the same K steps again with library-owned CUDA
    # events around every launch.  Events between launches forgo the
    # programmatic-launch overlap of neighbouring kernels, so this pass only
    # feeds the per-kernel shares and the roofline; `value` is the pass above.
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    with h3b.Trace(capacity=args.steps * (4000 if loop else 16 * len(blocks) + 8)) as tr:
        t0.record(stream)
        for _ in range(args.steps):
            eager_step()
        t1.record(stream)
        torch.cuda.synchronize()
    _barrier(world)
    clocks = sampler.stop()
    ms_traced = max_over_ranks(t0.elapsed_time(t1), dev)
    assert h3b.device_error() == 0, "device error word set during the timed region"

    # per-kernel shares from the live trace
    per = tr.by_kernel()
    total_k = sum(s for _, s in per.values()) or 1.0
    kernels = {k: {"launches": c, "ms_total": round(s, 4), "share": round(s / total_k, 4)} for k, (c, s) in
               sorted(per.items(), key=lambda kv: -kv[1][1])}
    my_launches = sum(c for k, (c, _) in per.items() if k != "memset")
    pk, src = peaks()
    bf16_pk = tensor_peak(pk, clocks, int8=False)
    int8_pk = tensor_peak(pk, clocks, int8=True)
    dom = max(per.items(), key=lambda kv: kv[1][1])[0]
    amount, unit, bound = kernel_work(dom, wl, wl.dtype)
    if loop and wl.merge_first >= 0 and bound == "tensor":
        n_m = wl.merge_last - wl.merge_first + 1
        amount_m, _, _ = kernel_work(dom, wl, wl.dtype, merged=True)
        amount = ((wl.n_blocks - n_m) * amount + n_m * amount_m) / wl.n_blocks
    roof = None
    if amount is not None:
        avg_s = per[dom][1] / per[dom][0] / 1e3
        if bound == "tensor":
            tp = int8_pk if unit == "TOP/s" else bf16_pk
            peak, basis, nominal = tp["peak"], tp["basis"], tp["nominal"]
            achieved = amount / avg_s / 1e12
        else:
            peak, basis, nominal = pk.get("hbm_gbs"), f"{src} copy bandwidth", NOMINAL["hbm_gbs"]
            achieved = amount / avg_s / 1e9
        roof = {"kernel": dom, "bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": unit,
                "frac": round(achieved / peak, 4), "traffic": measured_traffic(dom, wl.name),
                "peak_basis": basis, "frac_nominal": round(achieved / nominal, 4), "nominal_peak": nominal,
                "work_per_launch": amount, "avg_launch_ms": round(avg_s * 1e3, 4)}

    value = whole_job_value(units, args.steps, world, ms)
    if loop:
        metric, unit_v, hib = "s per denoise step", "s/step", False
        value = ms / 1e3 / args.steps / wl.steps
    else:
        metric, unit_v, hib = METRIC, "tokens/s", True
    flops_step = wl.block_flops() * (len(blocks) if not loop else 0)
    if loop:
        fm, fr = wl.merge_first, wl.merge_last
        fl = wl.with_(n_audio=wl.n_audio + args.cond_rows)  # condition rows add to every block's sequence
        if core:
            outer = sum(fl.block_flops() for l in range(len(blocks)) if not fm <= l <= fr)
            inner = sum(fl.block_flops(merged=True) for l in range(fm, fr + 1))
            flops_step = outer * n_fresh + inner * n_core
        else:
            per_eval = sum(fl.block_flops(merged=(fm >= 0 and fm <= l <= fr)) for l in range(len(blocks)))
            flops_step = per_eval * n_fresh

    # Whole-step roofline: every launch's algorithmic work at its own bound's
    # peak (tensor peaks chosen for the sampled clock), summed over the step,
    # against the untraced step time.
    if not loop:
        t_ideal = t_nominal = 0.0
        for k, (c, _) in per.items():
            a, u, b = kernel_work(k, wl, wl.dtype)
            if a is None:
                continue
            if b == "tensor":
                i8 = u == "TOP/s"
                t_ideal += c * a / ((int8_pk if i8 else bf16_pk)["peak"] * 1e12)
                t_nominal += c * a / ((NOMINAL["int8_tops"] if i8 else NOMINAL["bf16_tflops"]) * 1e12)
            else:
                t_ideal += c * a / (pk.get("hbm_gbs") * 1e9)
                t_nominal += c * a / (NOMINAL["hbm_gbs"] * 1e9)
        t_ideal /= args.steps
        t_nominal /= args.steps
        basis = ("every traced launch: GEMM/attention work at the clock-chosen tensor peak "
                 f"(bf16 {bf16_pk['peak']:.0f} TF/s, int8 {int8_pk['peak']:.0f} TOP/s), memory kernels at the "
                 f"{src} copy bandwidth")
    else:
        t_ideal = flops_step / (bf16_pk["peak"] * 1e12)
        t_nominal = flops_step / (NOMINAL["bf16_tflops"] * 1e12)
        basis = (f"GEMM + attention work of the step at the clock-chosen bf16 peak ({bf16_pk['peak']:.0f} TF/s; "
                 "memory-bound kernels < 2 %)")
    t_step = ms / 1e3 / args.steps
    step_roofline = {"t_ideal_ms": round(t_ideal * 1e3, 4), "t_ms": round(t_step * 1e3, 4),
                     "frac": round(t_ideal / t_step, 4), "frac_nominal": round(t_nominal / t_step, 4),
                     "basis": basis}

    # end-to-end through the public API with the tokens in pinned host memory:
    # every step copies its input in and its result out inside the timed
    # region; HostPipeline overlaps those copies with the neighbouring steps'
    # compute on separate streams.
    if not loop:
        k2 = max(4, min(args.steps, 50))
        xin = [x.detach().cpu().pin_memory() for _ in range(2)]
        xout = [torch.empty_like(xin[0]).pin_memory() for _ in range(2)]
        pipe = h3b.HostPipeline(dm, blocks, ws, tuple(x.shape))
        for i in range(4):
            pipe.submit(xin[i % 2], xout[i % 2])
        pipe.synchronize()
        torch.cuda.synchronize()
        _barrier(world)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(pipe.s_in)
        for i in range(k2):
            pipe.submit(xin[i % 2], xout[i % 2])
        f1.record(pipe.s_out)
        pipe.synchronize()
        torch.cuda.synchronize()
        _barrier(world)
        ms2 = max_over_ranks(f0.elapsed_time(f1), dev)
        nb = x.numel() * 4
        e2e = {"value": round(whole_job_value(units, k2, world, ms2), 2), "unit": unit_v, "h2d_bytes_per_step": nb,
               "d2h_bytes_per_step": nb, "steps": k2,
               "api": "h3b.HostPipeline.submit (pinned host in/out, copies overlapped with compute)"}
        del pipe
    else:
        # one step = one whole denoising loop: x0 comes in from pinned host
        # memory and x_N goes back to it inside the timed region
        k2 = max(1, min(args.steps, 2))
        xh = x.detach().cpu().pin_memory()
        xo = torch.empty_like(xh).pin_memory()
        torch.cuda.synchronize()
        _barrier(world)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(k2):
            x.copy_(xh, non_blocking=True)
            step()
            xo.copy_(x, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        _barrier(world)
        ms2 = max_over_ranks(f0.elapsed_time(f1), dev)
        nb = x.numel() * 4
        e2e = {"value": round(ms2 / 1e3 / k2 / wl.steps, 6), "unit": unit_v, "h2d_bytes_per_step": nb,
               "d2h_bytes_per_step": nb, "steps": k2,
               "api": "h3b.denoise / h3b.denoise_ex with x0 copied in from and x_N copied out to pinned host memory"}

    rec = {
        "metric": metric, "value": round(value, 6 if loop else 2), "unit": unit_v, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "ms_per_step_traced": round(ms_traced / args.steps, 4),
        "higher_is_better": hib, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 GEMMs / bf16 attention" if wl.dtype == W.INT8 else "bf16",
        "data": "synthetic (seeded N(0,0.02) bf16 weights, N(0,1) fp32 tokens)",
        "config": {"workload": wl.name, "seq_len": wl.seq, "d": wl.d, "heads": wl.n_heads,
                   "head_dim": wl.head_dim, "ffn": wl.ffn, "blocks": len(blocks),
                   "video_grid": [wl.frames, wl.rows, wl.cols], "audio_tokens": wl.n_audio,
                   "global_batch": 1, "parallelism": f"replicas x{world}",
                   "launch": "one CUDA graph replay per step" if args.graph else "eager (programmatic dependent launch)",
                   "l2": "no flush: per-step working set (weights + activations + workspace) > 126 MB L2"},
        "tflops": round(flops_step * args.steps * world / (ms / 1e3) / 1e12, 2),
        "roofline": roof, "step_roofline": step_roofline, "gpu_launches": my_launches, "clocks": clocks,
        "tensor_peaks": {"bf16": bf16_pk, "int8": int8_pk}, "kernels": kernels, "e2e": e2e,
    }
    if loop:
        rec["s_per_fresh_eval"] = round(ms / 1e3 / args.steps / n_fresh, 6)
        rec["config"].update({"steps": wl.steps, "reuse": 1 if core else wl.reuse, "fresh_evals": n_fresh,
                              "token_reduction": [wl.merge_first, wl.merge_last],
                              "unmerge": "delta" if args.unmerge_delta else "broadcast"})
        if core:
            rec["config"].update({"core_reuse": args.core_reuse, "core_blocks": [wl.merge_first, wl.merge_last],
                                  "core_evals": n_core})
        if args.cond_rows or args.modulation:
            rec["config"].update({"cond_rows": args.cond_rows, "modulation": "per step" if args.modulation else None})
        rec["ms_per_loop"] = round(ms / args.steps, 3)
    del blocks, x, ws, v
    torch.cuda.empty_cache()
    return rec


def run_ours(args, wl):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    line = measure(args, wl, dev, world, local)
    # The INT8 W8A8 block (d = 5120 over 5x48x84 video + 480 audio tokens) is
    # timed in the same run with the same protocol, as a sub-record.
    if args.workload == DEFAULT_WORKLOAD and not args.no_int8 and not (args.layers or args.denoise_steps):
        sub = measure(args, W.WORKLOADS[INT8_WORKLOAD], dev, world, local)
        line["int8"] = {k: sub[k] for k in ("metric", "value", "unit", "ms_per_step", "ms_per_step_traced",
                                            "dtype", "config", "tflops", "roofline", "step_roofline",
                                            "gpu_launches", "clocks", "tensor_peaks", "kernels", "e2e")}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- CPU oracle
def _oracle_inputs(wl, layer=0):
    w = {k: v.float().numpy() for k, v in W.block_weights(wl, layer, "cpu").items()}
    x = W.initial_tokens(wl, "cpu").numpy()
    return w, x


class OracleChunks:
    """The oracle block (fp64 numpy) run one token chunk at a time.

    Chunk i of n takes its tokens through every part of the block -- RMSNorm,
    the Q, K and V projections of those tokens, RoPE, attention of its
    queries against all S keys and values, O-projection + residual, RMSNorm,
    GELU MLP + residual -- and writes its K and V rows into a cache that holds
    all S tokens' keys and values (filled once at set-up).  Each chunk is thus
    1/n of the block's arithmetic, and n consecutive chunks are exactly one
    block's work: the time of one chunk is the time behind (S/n) tokens of
    block throughput.  Only the oracle's own functions are called."""

    def __init__(self, wl, n_chunks=8):
        import oracle
        self.o = oracle
        self.wl = wl
        w, x = _oracle_inputs(wl)
        if wl.dtype == W.INT8:
            w = oracle.dequant_weights(w)  # the INT8 parity reference: dequantised weights
        self.w = {k: np.asarray(v, dtype=np.float64) for k, v in w.items()}
        self.x = np.asarray(x, dtype=np.float64)
        self.ang = oracle.rope_angles(wl)
        d = wl.d
        u = oracle.rmsnorm(self.x, self.w["g_attn"], wl.eps)
        self.k = oracle.apply_rope(oracle.linear(u, self.w["w_qkv"][d:2 * d]), self.ang, wl.n_heads)
        self.v = oracle.linear(u, self.w["w_qkv"][2 * d:])
        self.bounds = np.linspace(0, wl.seq, n_chunks + 1).astype(int)
        self.n = n_chunks

    def run(self, i):
        o, wl, w, d = self.o, self.wl, self.w, self.wl.d
        lo, hi = self.bounds[i % self.n], self.bounds[i % self.n + 1]
        x = self.x[lo:hi]
        u = o.rmsnorm(x, w["g_attn"], wl.eps)
        qkv = o.linear(u, w["w_qkv"])
        q = o.apply_rope(qkv[:, :d], self.ang[lo:hi], wl.n_heads)
        self.k[lo:hi] = o.apply_rope(qkv[:, d:2 * d], self.ang[lo:hi], wl.n_heads)
        self.v[lo:hi] = qkv[:, 2 * d:]
        x1 = x + o.linear(o.attention(q, self.k, self.v, wl.n_heads), w["w_o"])
        g = o.gelu(o.linear(o.rmsnorm(x1, w["g_mlp"], wl.eps), w["w_fc1"]))
        return x1 + o.linear(g, w["w_fc2"])

    def tokens(self, i):
        return int(self.bounds[i % self.n + 1] - self.bounds[i % self.n])


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 0) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl, budget_s=20.0, n_chunks=8):
    """Block tokens/s of the oracle on this host: whole 1/n-block chunks
    (OracleChunks) until about budget_s seconds of CPU work, at least two."""
    oc = OracleChunks(wl, n_chunks)
    oc.run(0)  # warm-up (BLAS threads, page-in)
    done = toks = 0
    t0 = time.perf_counter()
    while done < 2 or (time.perf_counter() - t0 < budget_s and done < n_chunks):
        oc.run(done)
        toks += oc.tokens(done)
        done += 1
    dt = time.perf_counter() - t0
    sample = (f"{done} of the {n_chunks} token chunks of one {wl.name} block (layer 0; the stack's blocks share its "
              f"shape), each chunk through the whole block in fp64 numpy with attention against all {wl.seq} keys: "
              f"{toks} tokens in {dt:.1f} s")
    if wl.steps > 0:
        per_block = dt / toks * wl.seq
        n_fresh = len([i for i in range(wl.steps) if i % wl.reuse == 0 or i == wl.steps - 1])
        return {"value": round(per_block * wl.n_blocks * n_fresh / wl.steps, 3), "unit": "s/step",
                "cores": cpu_threads(), "cpu_model": cpu_model(), "kind": "oracle",
                "sample": sample + f"; extrapolated to {wl.n_blocks} full-length blocks x {n_fresh} fresh "
                                   f"evaluations / {wl.steps} steps (merged blocks counted at full length)"}
    return {"value": round(toks / dt, 3), "unit": "tokens/s", "cores": cpu_threads(), "cpu_model": cpu_model(),
            "kind": "oracle", "sample": sample}


def run_reference(args, wl):
    """The oracle as the reference arm: one step = one 1/8-block token chunk of
    the workload (OracleChunks), so eight steps are one block's arithmetic and
    `value` = chunk tokens / chunk time (block tokens/s, the same unit as our
    arm's).  Set-up (weights, the K/V cache) is untimed."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    if wl.steps > 0:
        print(json.dumps({"impl": "reference", "unavailable": "the loop workloads are reported through their "
                                                              "extrapolated cpu_baseline only"}), flush=True)
        return
    oc = OracleChunks(wl, 8)
    for i in range(args.warmup):
        oc.run(i)
    toks = 0
    t0 = time.perf_counter()
    for i in range(args.steps):
        oc.run(i)
        toks += oc.tokens(i)
    dt = time.perf_counter() - t0
    value = toks / dt
    sample = (f"each step: one of the 8 token chunks of a {wl.name} block (about {wl.seq // 8} tokens) through the "
              f"whole block in fp64 numpy, attention against all {wl.seq} keys; 8 steps = one block's arithmetic; "
              f"{toks} tokens in {dt:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (same seeded inputs)",
            "config": {"workload": wl.name, "seq_len": wl.seq, "d": wl.d, "heads": wl.n_heads,
                       "head_dim": wl.head_dim, "ffn": wl.ffn, "blocks": wl.n_blocks,
                       "video_grid": [wl.frames, wl.rows, wl.cols], "audio_tokens": wl.n_audio,
                       "global_batch": 1, "parallelism": "cpu"},
            "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cpu_threads(),
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- peak and kernel probes
def measure_int8_peak(out_path, n=8192, burst_reps=10, sustain_s=4.0):
    """Dense int8 tensor peak of this GPU, the way the bf16 peaks are taken:
    torch._int_mm (cuBLAS) on n^3, best of burst_reps single launches (CUDA
    events), then back-to-back launches for sustain_s seconds with the SM
    clock sampled; bf16 torch.matmul on the same box for the ratio."""
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    a = torch.randint(-127, 128, (n, n), generator=g, device=dev, dtype=torch.int8)
    b = torch.randint(-127, 128, (n, n), generator=g, device=dev, dtype=torch.int8).t()  # column-major
    ab = torch.randn((n, n), generator=g, device=dev).to(torch.bfloat16)
    bb = torch.randn((n, n), generator=g, device=dev).to(torch.bfloat16)
    ops = 2.0 * n ** 3

    def burst(fn):
        for _ in range(3):
            fn()
        best = None
        for _ in range(burst_reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / 1e3
            best = t if best is None else min(best, t)
        return ops / best / 1e12

    def sustained(fn):
        sampler = ClockSampler(0)
        fn()
        torch.cuda.synchronize()
        t_est = max(1e-4, ops / (burst_i8 * 1e12))
        reps = max(10, int(sustain_s / t_est))
        sampler.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        clocks = sampler.stop()
        return ops * reps / (e0.elapsed_time(e1) / 1e3) / 1e12, clocks, reps

    i8 = lambda: torch._int_mm(a, b)  # noqa: E731
    bf = lambda: torch.matmul(ab, bb)  # noqa: E731
    burst_i8 = burst(i8)
    burst_bf = burst(bf)
    sust_i8, clk, reps = sustained(i8)
    rec = {"int8_tops": round(burst_i8, 1), "int8_tops_sustained": round(sust_i8, 1),
           "sustained_sm_mhz_median": clk.get("sm_mhz"), "sustained_clocks": clk,
           "bf16_tflops_same_box": round(burst_bf, 1), "int8_over_bf16_burst": round(burst_i8 / burst_bf, 3),
           "gpu": torch.cuda.get_device_name(dev), "torch": torch.__version__,
           "how": (f"torch._int_mm int8 {n}^3 (A row-major, B column-major; 2*n^3 ops): best of {burst_reps} "
                   f"(CUDA events) and {reps} back-to-back launches with nvidia-smi clock samples; "
                   f"torch.matmul bf16 {n}^3 best of {burst_reps} on the same box"),
           "when": datetime.datetime.now(datetime.timezone.utc).strftime("%Y-%m-%dT%H:%M:%SZ"),
           "command": "python bench.py --measure-int8-peak"}
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    with open(out_path, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec), flush=True)


def library_compare(args):
    """This library's GEMMs and attention against the vendor libraries on the
    d = 5120 shapes, timed back to back on one GPU in alternating rounds
    (CUDA events, median): the four linear layers with a plain bf16 output
    against torch.matmul (cuBLAS, same operand layouts, no K split here), and
    bidirectional attention against torch's scaled_dot_product_attention with
    the cuDNN and flash backends, on strided views of the same qkv buffer.
    The implementations of a case run in interleaved blocks whose order
    alternates, so both see the same clock history under the power cap; the
    figure is the median over the blocks.  A comparison only: nothing on the
    product path calls these libraries.  One JSON line per case."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    from audio_diffusion_transformer_dit_b200 import h3b
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    def interleaved(fns, blocks=8, group=5):
        for fn in fns.values():
            for _ in range(3):
                fn()
        torch.cuda.synchronize()
        ts = {k: [] for k in fns}
        for b in range(blocks):
            for k in (list(fns) if b % 2 == 0 else list(fns)[::-1]):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(group):
                    fns[k]()
                e1.record()
                torch.cuda.synchronize()
                ts[k].append(e0.elapsed_time(e1) / group)
        return {k: statistics.median(v) for k, v in ts.items()}

    wl = W.WORKLOADS["stack8_d5120_s6528"]
    S, d, f = wl.seq, wl.d, wl.ffn
    gemms = {"qkv": (S, 3 * d, d), "o_proj": (S, d, d), "fc1": (S, f, d), "fc2": (S, d, f)}
    attn = [(S, wl.n_heads), (6400, 24), (W.WORKLOADS[INT8_WORKLOAD].seq, wl.n_heads)]
    only = set(args.sweep_only.split(",")) if args.sweep_only else None
    for name, (M, N, K) in gemms.items():
        if only and name not in only:
            continue
        A = W.normal_tensor((M, K), 1, dev, dtype=torch.bfloat16)
        B = W.normal_tensor((N, K), 2, dev, 0.02, dtype=torch.bfloat16)
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        clk = ClockSampler(0)
        clk.start()
        t = interleaved({"ours": lambda: h3b.gemm(A, B, h3b.EPI_BF16, C),
                         "cublas": lambda: torch.matmul(A, B.t(), out=C)})
        clocks = clk.stop()
        fl = 2.0 * M * N * K
        print(json.dumps({"compare": "gemm_bf16", "case": name, "shape_mnk": [M, N, K], "clocks": clocks,
                          **{f"{k}_ms": round(v, 4) for k, v in t.items()},
                          **{f"{k}_tflops": round(fl / v / 1e9, 1) for k, v in t.items()},
                          "ours_over_cublas_speed": round(t["cublas"] / t["ours"], 3)}), flush=True)
        del A, B, C
    for Sa, H in attn:
        name = f"attention_s{Sa}_h{H}"
        if only and name not in only:
            continue
        D = wl.head_dim
        qkv = W.normal_tensor((Sa, 3 * H * D), 25, dev, dtype=torch.bfloat16)
        scr = torch.empty(2 * Sa * H * D, dtype=torch.float32, device=dev)
        out = torch.empty((Sa, H * D), dtype=torch.bfloat16, device=dev)
        q, k, v = (qkv[:, i * H * D:(i + 1) * H * D].view(Sa, H, D).transpose(0, 1).unsqueeze(0) for i in range(3))
        fl = 4.0 * Sa * Sa * H * D

        def sdpa(be):
            def run():
                with sdpa_kernel(be):
                    return F.scaled_dot_product_attention(q, k, v)
            return run
        fns = {"ours": lambda: h3b.attention(qkv, H, D, o=out, scratch=scr)}
        rec = {"compare": "attention", "case": name}
        for bname, be in (("cudnn", SDPBackend.CUDNN_ATTENTION), ("flash", SDPBackend.FLASH_ATTENTION)):
            try:
                r = sdpa(be)()[0].transpose(0, 1).reshape(Sa, H * D)
                fns["ours"]()
                torch.cuda.synchronize()
                rec[f"{bname}_max_abs_diff"] = float((r.float() - out.float()).abs().max())
                fns[bname] = sdpa(be)
            except RuntimeError as e:  # backend not available for this shape or build
                rec[f"{bname}_error"] = str(e).splitlines()[0][:160]
        clk = ClockSampler(0)
        clk.start()
        t = interleaved(fns, group=2 if Sa > 10000 else 5)
        rec["clocks"] = clk.stop()
        rec.update({f"{k}_ms": round(v, 4) for k, v in t.items()})
        rec.update({f"{k}_tflops": round(fl / v / 1e9, 1) for k, v in t.items()})
        rec.update({f"ours_over_{k}_speed": round(v / t["ours"], 3) for k, v in t.items() if k != "ours"})
        print(json.dumps(rec), flush=True)
        del qkv, scr, out, q, k, v


def kernel_sweep(args):
    """Each memory-bound kernel of the path timed alone at the d = 5120
    workload sizes (CUDA events, median of the repetitions; every input is
    larger than L2, so no flush is needed; outputs come from torch's caching
    allocator, which launches nothing): algorithmic bytes, time, GB/s and the
    fraction of the measured copy bandwidth.  One JSON line per kernel."""
    from audio_diffusion_transformer_dit_b200 import h3b
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pk, src = peaks()
    hbm = pk.get("hbm_gbs")
    wl4 = W.WORKLOADS[INT8_WORKLOAD]  # 20640 tokens x 5120, MLP 20480
    wl5 = W.WORKLOADS["loop45_d5120_s6528"]  # 6528 tokens, merge 6144 -> 3072 video tokens
    S, d, f = wl4.seq, wl4.d, wl4.ffn
    x = W.normal_tensor((S, d), 11, dev)
    g = torch.ones(d, dtype=torch.float32, device=dev)
    abf = W.normal_tensor((S, d), 12, dev, dtype=torch.bfloat16)
    gbf = W.normal_tensor((S, f), 13, dev, dtype=torch.bfloat16)
    amax = gbf.float().abs().amax(dim=1).contiguous()
    dm5 = h3b.dims_of(wl5)
    x5 = W.normal_tensor((wl5.seq, wl5.d), 14, dev)
    xm5 = torch.empty((wl5.seq_merged, wl5.d), dtype=torch.float32, device=dev)
    v5 = W.normal_tensor((wl5.seq, wl5.d), 15, dev)
    cp5 = torch.empty_like(v5)
    ym5 = W.normal_tensor((wl5.seq_merged, wl5.d), 16, dev)
    # outputs allocated once: every timed launch is the library call alone
    u_bf = torch.empty((S, d), dtype=torch.bfloat16, device=dev)
    q_d = torch.empty((S, d), dtype=torch.int8, device=dev)
    q_f = torch.empty((S, f), dtype=torch.int8, device=dev)
    s_r = torch.empty(S, dtype=torch.float32, device=dev)
    lib, st = h3b.lib, h3b._stream()
    P = lambda t: t.data_ptr()  # noqa: E731
    cases = [
        ("rmsnorm_bf16", lambda: lib.h3b_rmsnorm(P(x), P(g), S, d, 1e-6, P(u_bf), None, h3b.BF16, st),
         S * d * 4 + S * d * 2, f"x fp32 [{S},{d}] -> bf16"),
        ("rmsnorm_int8", lambda: lib.h3b_rmsnorm(P(x), P(g), S, d, 1e-6, P(q_d), P(s_r), h3b.INT8, st),
         S * d * 4 + S * d + S * 4, f"x fp32 [{S},{d}] -> int8 + scale"),
        ("quant_rows", lambda: lib.h3b_quantize_weights(P(abf), S, d, P(q_d), P(s_r), st),
         S * d * 2 + S * d + S * 4, f"o bf16 [{S},{d}] -> int8 + scale"),
        ("quant_absmax", lambda: lib.h3b_quantize_rows_absmax(P(gbf), P(amax), S, f, P(q_f), P(s_r), st),
         S * f * 2 + S * f + S * 8, f"g bf16 [{S},{f}] + row max -> int8 + scale"),
        ("token_merge", lambda: lib.h3b_token_merge(ctypes.byref(dm5), P(x5), P(xm5), st),
         (wl5.seq + wl5.seq_merged) * wl5.d * 4, f"x fp32 [{wl5.seq},{wl5.d}] -> [{wl5.seq_merged},{wl5.d}]"),
        ("token_unmerge", lambda: lib.h3b_token_unmerge(ctypes.byref(dm5), P(xm5), P(x5), st),
         (wl5.seq + wl5.seq_merged) * wl5.d * 4, f"xm fp32 [{wl5.seq_merged},{wl5.d}] -> [{wl5.seq},{wl5.d}]"),
        ("token_unmerge_delta", lambda: lib.h3b_token_unmerge_delta(ctypes.byref(dm5), P(x5), P(ym5), P(xm5), st),
         2 * (wl5.seq + wl5.seq_merged) * wl5.d * 4,
         f"x fp32 [{wl5.seq},{wl5.d}] += (ym - xm0) [{wl5.seq_merged},{wl5.d}] broadcast"),
        ("flow_step", lambda: lib.h3b_flow_step(P(x5), P(v5), ctypes.c_float(0.5), ctypes.c_float(0.45),
                                                 ctypes.c_size_t(x5.numel()), None, st),
         3 * wl5.seq * wl5.d * 4, f"x, v fp32 [{wl5.seq},{wl5.d}] -> x"),
        ("flow_step_copy", lambda: lib.h3b_flow_step(P(x5), P(v5), ctypes.c_float(0.5), ctypes.c_float(0.45),
                                                      ctypes.c_size_t(x5.numel()), P(cp5), st),
         4 * wl5.seq * wl5.d * 4, f"x, v fp32 [{wl5.seq},{wl5.d}] -> x and a copy"),
    ]
    only = set(args.sweep_only.split(",")) if args.sweep_only else None
    # contractions, timed alone: the INT8 and BF16 FC1 GEMMs (GELU epilogue;
    # INT8 also writes the per-row max), the FC2 and O-projection GEMMs
    # (fp32 residual epilogue) and the attention of the d = 3072 block and
    # both d = 5120 workloads; built only when selected (they hold ~1-3 GB)
    tensor_cases = {
        "gemm_fc1_int8": (INT8_WORKLOAD, "int8"), "gemm_fc1_bf16": (DEFAULT_WORKLOAD, "bf16"),
        "gemm_fc2_bf16": (DEFAULT_WORKLOAD, "bf16"),
        "gemm_o_bf16_d3072": ("block_d3072_s6400", "bf16"), "gemm_o_bf16_d5120": (DEFAULT_WORKLOAD, "bf16"),
        "attention_s6400": ("block_d3072_s6400", None), "attention_s6528": (DEFAULT_WORKLOAD, None),
        "attention_s20640": (INT8_WORKLOAD, None),
    }
    for name, (wname, kind) in tensor_cases.items():
        if only is None or name not in only:
            continue
        wl = W.WORKLOADS[wname]
        Sx, dx, fx = wl.seq, wl.d, wl.ffn
        if name == "gemm_fc2_bf16":  # x [S, d] fp32 += g [S, f] W2 [d, f]^T
            A = W.normal_tensor((Sx, fx), 21, dev, dtype=torch.bfloat16)
            B = W.normal_tensor((dx, fx), 22, dev, std=0.02, dtype=torch.bfloat16)
            C = W.normal_tensor((Sx, dx), 23, dev)
            fn = lambda A=A, B=B, C=C: h3b.gemm(A, B, h3b.EPI_RESID, C)  # noqa: E731
            work = 2.0 * Sx * fx * dx
            shape = f"bf16 [{Sx},{fx}] x [{dx},{fx}]^T -> fp32 residual [{Sx},{dx}]"
        elif name.startswith("gemm_o"):  # x [S, d] fp32 += o [S, d] Wo [d, d]^T, tail split along K
            A = W.normal_tensor((Sx, dx), 21, dev, dtype=torch.bfloat16)
            B = W.normal_tensor((dx, dx), 22, dev, std=0.02, dtype=torch.bfloat16)
            C = W.normal_tensor((Sx, dx), 23, dev)
            scr = torch.empty(Sx * dx, dtype=torch.float32, device=dev)
            fn = lambda A=A, B=B, C=C, scr=scr: h3b.gemm(A, B, h3b.EPI_RESID, C, scratch=scr)  # noqa: E731
            work = 2.0 * Sx * dx * dx
            shape = f"bf16 [{Sx},{dx}] x [{dx},{dx}]^T -> fp32 residual [{Sx},{dx}]"
        elif name.startswith("gemm"):
            if kind == "int8":
                A = W.int8_tensor((Sx, dx), 21, dev)
                B = W.int8_tensor((fx, dx), 22, dev)
                sa = W.uniform_tensor((Sx,), 23, dev, 1e-3, 2e-3)
                sb = W.uniform_tensor((fx,), 24, dev, 1e-3, 2e-3)
            else:
                A = W.normal_tensor((Sx, dx), 21, dev, dtype=torch.bfloat16)
                B = W.normal_tensor((fx, dx), 22, dev, std=0.02, dtype=torch.bfloat16)
                sa = sb = None
            C = torch.empty((Sx, fx), dtype=torch.bfloat16, device=dev)
            rmax = torch.zeros(Sx, dtype=torch.float32, device=dev) if kind == "int8" else None
            fn = (lambda A=A, B=B, C=C, sa=sa, sb=sb, rmax=rmax:
                  h3b.gemm(A, B, h3b.EPI_GELU, C, scale_a=sa, scale_b=sb, row_absmax=rmax))
            work = 2.0 * Sx * fx * dx
            shape = f"{kind} [{Sx},{dx}] x [{fx},{dx}]^T -> GELU bf16"
        else:
            qkv = W.normal_tensor((Sx, 3 * dx), 25, dev, dtype=torch.bfloat16)
            o = torch.empty((Sx, dx), dtype=torch.bfloat16, device=dev)
            scr = torch.empty(2 * Sx * dx, dtype=torch.float32, device=dev)
            fn = (lambda qkv=qkv, o=o, scr=scr, wl=wl:
                  h3b.attention(qkv, wl.n_heads, wl.head_dim, o=o, scratch=scr))
            work = 4.0 * Sx * Sx * dx
            shape = f"bf16 S={Sx}, {wl.n_heads} heads x {wl.head_dim}"
        cases.append((name, fn, work, shape))
    for name, fn, amount, shape in cases:
        if only and name not in only:
            continue
        tensor = name in tensor_cases
        for _ in range(args.sweep_warmup):
            rc = fn()
            assert not isinstance(rc, int) or rc == 0, f"{name}: status {rc}"
        torch.cuda.synchronize()
        assert h3b.device_error() == 0
        # back-to-back launches between two events (the launch latency of one
        # call hides behind the previous kernel), in groups; the median group
        group = max(1, args.sweep_group)
        times = []
        sampler = ClockSampler(0)
        sampler.start()
        for _ in range(max(1, args.sweep_reps // group)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(group):
                fn()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / group)
        clocks = sampler.stop()
        assert h3b.device_error() == 0
        t = statistics.median(times) / 1e3
        rec = {"kernel": name, "shape": shape, "us_median": round(t * 1e6, 2), "us_min": round(min(times) * 1e3, 2),
               "launches": group * len(times), "clocks": clocks}
        if tensor:
            tp = tensor_peak(pk, clocks, int8=name.endswith("int8"))
            rate = amount / t / 1e12
            rec.update({"work": amount, "unit": "TOP/s" if name.endswith("int8") else "TFLOP/s",
                        "achieved": round(rate, 1), "peak": tp["peak"], "frac": round(rate / tp["peak"], 4),
                        "peak_basis": tp["basis"], "frac_nominal": round(rate / tp["nominal"], 4)})
        else:
            rec.update({"bytes": amount, "gbs": round(amount / t / 1e9, 1), "frac": round(amount / t / 1e9 / hbm, 4),
                        "peak_gbs": hbm, "peak_source": src})
        print(json.dumps(rec), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-int8", action="store_true",
                    help="default workload: skip the INT8 d=5120 S=20640 block sub-record")
    ap.add_argument("--core-reuse", type=int, default=0,
                    help="loop workload: core residual reuse over the reduction window (replaces velocity reuse)")
    ap.add_argument("--unmerge-delta", action="store_true", help="loop workload: delta-broadcast unmerge")
    ap.add_argument("--layers", type=int, default=0,
                    help="loop workload: run only the first L blocks (the pages' --layers 40/45/50)")
    ap.add_argument("--denoise-steps", type=int, default=0,
                    help="loop workload: denoising steps (the pages' 4..7-step presets; default: the workload's)")
    ap.add_argument("--cond-rows", type=int, default=0,
                    help="loop workload: fixed condition rows appended after the audio tokens")
    ap.add_argument("--modulation", action="store_true",
                    help="loop workload: per-step, per-block timestep modulation (shift/scale/gate)")
    ap.add_argument("--measure-int8-peak", action="store_true",
                    help="measure the dense int8 tensor peak (torch._int_mm) and write profiles/int8_peak.json")
    ap.add_argument("--kernel-sweep", action="store_true",
                    help="time each memory-bound kernel alone at the d=5120 sizes (GB/s vs the copy bandwidth)")
    ap.add_argument("--sweep-only", default="", help="comma-separated kernel names for --kernel-sweep")
    ap.add_argument("--sweep-reps", type=int, default=50)
    ap.add_argument("--sweep-warmup", type=int, default=5)
    ap.add_argument("--sweep-group", type=int, default=10, help="back-to-back launches per timed group")
    ap.add_argument("--graph", action="store_true",
                    help="capture the step into a CUDA graph once and time its replays")
    ap.add_argument("--library-compare", action="store_true",
                    help="time the GEMMs and attention against cuBLAS / cuDNN on the d=5120 shapes (comparison only)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # never fewer than 3 warm-up steps
    if args.library_compare:
        library_compare(args)
        return
    if args.measure_int8_peak:
        measure_int8_peak(INT8_PEAK_FILE)
        return
    if args.kernel_sweep:
        kernel_sweep(args)
        return
    wl = W.WORKLOADS[args.workload]
    if (args.layers or args.denoise_steps or args.cond_rows or args.modulation or args.core_reuse
            or args.unmerge_delta) and wl.steps == 0:
        ap.error("--layers, --denoise-steps, --cond-rows, --modulation, --core-reuse and --unmerge-delta apply to "
                 "the denoising-loop workloads")
    if args.layers or args.denoise_steps:
        if args.layers and not (0 < args.layers and (wl.merge_last < args.layers)):
            ap.error("--layers must keep the token-reduction window inside the active blocks")
        wl = wl.with_(n_blocks=args.layers or wl.n_blocks, steps=args.denoise_steps or wl.steps)
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload] if args.impl == "ours" else 10
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
