#!/usr/bin/env python
"""Benchmark of the DiT block hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the hot path over one batch of synthetic input.  The
default workload is the single bf16 DiT block d=3072 (24 heads x 128, MLP
12288) over 6x32x32 video + 256 audio tokens (S = 6400): one step is one
h3b_block_forward (RoPE table, RMSNorm, QKV GEMM + RoPE, flash attention,
O-proj + residual, RMSNorm, FC1 + GELU, FC2 + residual).  Other workloads:
the 8-block d=5120 stack, the INT8 W8A8 d=5120 block over 20640 tokens and the
45-block 20-step denoising loop with reuse 2 and token reduction.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize() on both sides, CUDA events on the launching stream,
max over ranks.  The working set (weights + activations + workspace) exceeds
the 126 MB L2, so no flush is inserted between steps.  N > 1 runs N
independent replicas (one per GPU, launched by torchrun); the path has no
exchange step, so there is no data-path collective ("scaling": "weak").
A second pass of the same K steps records library-owned CUDA events around
every launch for the per-kernel shares and the roofline of the dominant
kernel ("ms_per_step_traced"; the events between launches forgo the overlap
of neighbouring kernels, so `value` comes from the untraced pass).

--impl reference times the CPU oracle (numpy fp64) on the host cores on a
bounded sample of the same workload (rank 0 only under torchrun).
"""
from __future__ import annotations

import argparse
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

DEFAULT_WORKLOAD = "block_d3072_s6400"
METRIC = "DiT block tokens/s"
# default timed steps per workload: about 1-30 s of device time each
DEFAULT_STEPS = {"block_d256_s288": 2000, "block_d3072_s6400": 300, "stack8_d5120_s6528": 30,
                 "block_int8_d5120_s20640": 60, "loop45_d5120_s6528": 2,
                 "preview40_d5120_s2784": 4}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


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
              "flow_step": wl.seq * d * 4 * 3}
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


def run_ours(args, wl):
    from audio_diffusion_transformer_dit_b200 import h3b
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
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

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert h3b.device_error() == 0, "device error word set during warm-up"

    sampler = ClockSampler(local)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    # Per-kernel durations: the same K steps again with library-owned CUDA
    # events around every launch.  Events between launches forgo the
    # programmatic-launch overlap of neighbouring kernels, so this pass only
    # feeds the per-kernel shares and the roofline; `value` is the pass above.
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with h3b.Trace(capacity=args.steps * (4000 if loop else 16 * len(blocks) + 8)) as tr:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
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
            peak = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
            if unit == "TOP/s":
                peak = peak * 2.0  # int8 dense peak = bf16 measured x nominal ratio 4.5/2.25
            achieved = amount / avg_s / 1e12
        else:
            peak = pk.get("hbm_gbs")
            achieved = amount / avg_s / 1e9
        roof = {"kernel": dom, "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                "frac": round(achieved / peak, 4), "traffic": measured_traffic(dom, wl.name),
                "peak_source": f"{src} ({'sustained bf16' if bound == 'tensor' else 'copy'})",
                "work_per_launch": amount}

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
    # measured peak, summed over the step, against the untraced step time.
    tensor_peak = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    if not loop:
        t_ideal = 0.0
        for k, (c, _) in per.items():
            a, u, b = kernel_work(k, wl, wl.dtype)
            if a is None:
                continue
            if b == "tensor":
                t_ideal += c * a / (tensor_peak * (2.0 if u == "TOP/s" else 1.0) * 1e12)
            else:
                t_ideal += c * a / (pk.get("hbm_gbs") * 1e9)
        t_ideal /= args.steps
        basis = "every traced launch: GEMM/attention work at the sustained bf16 peak (int8 x2), memory kernels at HBM"
    else:
        t_ideal = flops_step / (tensor_peak * 1e12)
        basis = "GEMM + attention work of the step at the sustained bf16 peak (memory-bound kernels < 2 %)"
    t_step = ms / 1e3 / args.steps
    step_roofline = {"t_ideal_ms": round(t_ideal * 1e3, 4), "t_ms": round(t_step * 1e3, 4),
                     "frac": round(t_ideal / t_step, 4), "basis": basis}

    # end-to-end through the public API with the tokens in pinned host memory:
    # every step copies its input in and its result out inside the timed
    # region; HostPipeline overlaps those copies with the neighbouring steps'
    # compute on separate streams.
    e2e = None
    if not loop:
        k2 = max(4, min(args.steps, 50))
        xin = [x.detach().cpu().pin_memory() for _ in range(2)]
        xout = [torch.empty_like(xin[0]).pin_memory() for _ in range(2)]
        pipe = h3b.HostPipeline(dm, blocks, ws, tuple(x.shape))
        for i in range(4):
            pipe.submit(xin[i % 2], xout[i % 2])
        pipe.synchronize()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(pipe.s_in)
        for i in range(k2):
            pipe.submit(xin[i % 2], xout[i % 2])
        f1.record(pipe.s_out)
        pipe.synchronize()
        torch.cuda.synchronize()
        barrier()
        ms2 = max_over_ranks(f0.elapsed_time(f1), dev)
        nb = x.numel() * 4
        e2e = {"value": round(whole_job_value(units, k2, world, ms2), 2), "unit": unit_v, "h2d_bytes_per_step": nb,
               "d2h_bytes_per_step": nb, "steps": k2,
               "api": "h3b.HostPipeline.submit (pinned host in/out, copies overlapped with compute)"}
    else:
        # one step = one whole denoising loop: x0 comes in from pinned host
        # memory and x_N goes back to it inside the timed region
        k2 = max(1, min(args.steps, 2))
        xh = x.detach().cpu().pin_memory()
        xo = torch.empty_like(xh).pin_memory()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(k2):
            x.copy_(xh, non_blocking=True)
            step()
            xo.copy_(x, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms2 = max_over_ranks(f0.elapsed_time(f1), dev)
        nb = x.numel() * 4
        e2e = {"value": round(ms2 / 1e3 / k2 / wl.steps, 6), "unit": unit_v, "h2d_bytes_per_step": nb,
               "d2h_bytes_per_step": nb, "steps": k2,
               "api": "h3b.denoise / h3b.denoise_ex with x0 copied in from and x_N copied out to pinned host memory"}

    line = {
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
                   "l2": "no flush: per-step working set (weights + activations + workspace) > 126 MB L2"},
        "tflops": round(flops_step * args.steps * world / (ms / 1e3) / 1e12, 2),
        "roofline": roof, "step_roofline": step_roofline, "gpu_launches": my_launches, "clocks": clocks,
        "kernels": kernels,
    }
    if loop:
        line["s_per_fresh_eval"] = round(ms / 1e3 / args.steps / n_fresh, 6)
        line["config"].update({"steps": wl.steps, "reuse": 1 if core else wl.reuse, "fresh_evals": n_fresh,
                               "token_reduction": [wl.merge_first, wl.merge_last],
                               "unmerge": "delta" if args.unmerge_delta else "broadcast"})
        if core:
            line["config"].update({"core_reuse": args.core_reuse, "core_blocks": [wl.merge_first, wl.merge_last],
                                   "core_evals": n_core})
        if args.cond_rows or args.modulation:
            line["config"].update({"cond_rows": args.cond_rows, "modulation": "per step" if args.modulation else None})
        line["ms_per_loop"] = round(ms / args.steps, 3)
    if e2e:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- CPU oracle
def _oracle_inputs(wl, layer=0, merged=False):
    w = {k: v.float().numpy() for k, v in W.block_weights(wl, layer, "cpu").items()}
    x = W.initial_tokens(wl, "cpu", seq=wl.seq_merged if merged else wl.seq).numpy()
    return w, x


def oracle_block_rate(wl, rows_a=64, rows_b=256, reps=1):
    """Oracle block-forward time model on this host: T(R) = a + b R for R query
    rows (keys/values always cover all S tokens); returns (a, b, seconds used)."""
    import oracle
    w, x = _oracle_inputs(wl)
    if wl.dtype == W.INT8:
        w = oracle.dequant_weights(w)
    t_used = 0.0
    times = {}
    for R in (rows_a, rows_b):
        rows = np.linspace(0, wl.seq - 1, R).astype(int)
        best = None
        for _ in range(reps):
            t0 = time.perf_counter()
            oracle.block_forward(x, w, wl, rows=rows)
            dt = time.perf_counter() - t0
            t_used += dt
            best = dt if best is None else min(best, dt)
        times[R] = best
    b = max((times[rows_b] - times[rows_a]) / (rows_b - rows_a), 0.0)
    a = max(times[rows_a] - b * rows_a, 0.0)
    return a, b, t_used


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


def cpu_baseline(wl, budget_s=30.0):
    a, b, used = oracle_block_rate(wl)
    per_block = a + b * wl.seq
    n_blocks = wl.n_blocks
    if wl.steps > 0:
        n_fresh = len([i for i in range(wl.steps) if i % wl.reuse == 0 or i == wl.steps - 1])
        seconds = per_block * n_blocks * n_fresh / wl.steps
        return {"value": round(seconds, 3), "unit": "s/step", "cores": cpu_threads(), "cpu_model": cpu_model(),
                "kind": "oracle",
                "sample": f"oracle block forward on this host with 64 and 256 query rows (all {wl.seq} keys); "
                          f"full block {per_block:.2f} s extrapolated linearly in rows, x{n_blocks} blocks "
                          f"x{n_fresh} fresh evals / {wl.steps} steps (merged blocks counted at full S); "
                          f"{used:.1f} s of CPU time"}
    value = wl.seq / per_block
    return {"value": round(value, 3), "unit": "tokens/s", "cores": cpu_threads(), "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"oracle block forward (fp64 numpy) with 64 and 256 sampled query rows, keys/values over "
                      f"all {wl.seq} tokens; full-block time {per_block:.2f} s = fixed + per-row cost x {wl.seq} "
                      f"rows, fitted from the two runs ({used:.1f} s of CPU time)"}


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w, x = _oracle_inputs(wl)
    if wl.dtype == W.INT8:
        w = oracle.dequant_weights(w)
    # the fixed (keys/values) + per-row cost model, fitted during warm-up
    R = 64
    rows = np.linspace(0, wl.seq - 1, R).astype(int)
    a, b, _ = oracle_block_rate(wl)
    for _ in range(args.warmup):
        oracle.block_forward(x, w, wl, rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.block_forward(x, w, wl, rows=rows)
    dt = (time.perf_counter() - t0) / args.steps
    per_block = dt + b * (wl.seq - R)
    units = wl.seq * max(1, wl.n_blocks if wl.steps == 0 else 1)
    blocks = wl.n_blocks
    if wl.steps > 0:
        n_fresh = len([i for i in range(wl.steps) if i % wl.reuse == 0 or i == wl.steps - 1])
        value, unit, hib, metric = per_block * blocks * n_fresh / wl.steps, "s/step", False, "s per denoise step"
    else:
        value, unit, hib, metric = units / (per_block * blocks), "tokens/s", True, METRIC
    sample = (f"each step: oracle block forward (fp64 numpy), {R} sampled query rows against all {wl.seq} "
              f"keys/values; full block = step time + {wl.seq - R} rows x fitted per-row cost {b * 1e3:.3f} ms")
    line = {"impl": "reference", "metric": metric, "value": round(value, 4), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2),
            "higher_is_better": hib, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (same seeded inputs)", "config": {"workload": wl.name, "seq_len": wl.seq,
                                                                 "d": wl.d, "blocks": blocks},
            "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": cpu_threads(),
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
    ap.add_argument("--cpu-budget", type=float, default=30.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # never fewer than 3 warm-up steps
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
