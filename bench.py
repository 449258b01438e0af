#!/usr/bin/env python
"""MuonH optimizer-step benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen3_1.7b|qwen3_0.6b|single_256x512|sweep_<rows>x<cols>]
                    [--ns-precision fp16|bf16|fp32]

One step = one muonh_step over the whole matrix set (momentum, Newton-Schulz,
hyperball projection of every matrix).  Inputs are synthetic (W0 ~ N(0,0.02^2),
gradients ~ N(0,1e-3^2)), resident in HBM when the timed region starts, and
far larger than L2 (the 1.7B set moves ~34 GB of algorithmic traffic per
step), so no L2 flush is needed between steps.  With N > 1 (torchrun) every
rank runs an independent replica of the workload (no data-path collective);
the timed region is bracketed by barriers and the max over ranks is taken.

Rank 0 prints one JSON line.  --impl reference times the CPU oracle instead
(rank 0 only, no GPU work).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MuonH steps/s for Qwen3-1.7B matrix set on 1 B200; NS TFLOP/s & HBM GB/s vs peak"
UNIT = "steps/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# bytes per element actually moved by each elementwise kernel of this design
KERNEL_BYTES = {
    "momentum_norm": 14,   # read G, M; write M and the 16-bit Newton-Schulz input X
    "update_dots": 6,      # read W, 16-bit O
    "project": 10,         # read W, O; write W
}
# write_x only rewrites X for matrices whose momentum-kernel scale left the safe
# range (every matrix on the first step); it is timed but not given a GB/s.
ELEMENTWISE = ("momentum_norm", "write_x", "update_dots", "project")
# algorithmic bytes per element of the whole step (read G, M, W, O; write M, X, W)
ALGO_BYTES_PER_ELEM = 24


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3_1.7b")
    ap.add_argument("--ns-precision", default="fp16", choices=["fp16", "bf16", "fp32"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-aux", action="store_true")
    return ap.parse_args()


def workload_desc(name):
    import synth
    wl = synth.workload(name)
    shapes = [(m.rows, m.cols) for m in wl.matrices]
    return wl, shapes


def ns_flops(shapes, steps):
    """Dense-convention Newton-Schulz FLOPs: per iteration 4 r^2 c + 2 r^3."""
    tot = 0
    for rr, cc in shapes:
        r, c = min(rr, cc), max(rr, cc)
        tot += steps * (4 * r * r * c + 2 * r ** 3)
    return tot


def ns_flops_executed(shapes, steps, prec="fp16"):
    """Tensor-core FLOPs the Newton-Schulz kernels execute: GRAM and SQUARE
    run the tiles of the upper block triangle (256 x 256 CTA-pair tiles, or
    128 x 256 single-CTA tiles with three products each in FP32 mode), APPLY
    every tile of Y, all on the 256-padded buffers."""
    tm, mult = (128, 3) if prec == "fp32" else (256, 1)
    tot = 0
    for a, b in shapes:
        r = (min(a, b) + 255) // 256 * 256
        c = (max(a, b) + 255) // 256 * 256
        upper = sum(1 for bi in range(r // tm) for bj in range(r // 256) if bj * 256 + 255 >= bi * tm)
        tile = 2 * tm * 256
        tot += steps * mult * (upper * tile * c + upper * tile * r + (r // tm) * (c // 256) * tile * r)
    return tot


def apply_flops(shapes):
    """One APPLY pass over the set (Y' = aY + BY for every matrix): 2 r^2 c
    per matrix.  A step makes ns_steps such passes; a large set splits each
    pass into one launch per matrix group."""
    return sum(2 * min(a, b) ** 2 * max(a, b) for a, b in shapes)


def apply_bytes(shapes):
    """Algorithmic HBM bytes of one APPLY pass: read B' (r x r) and Y (r x c),
    write Y', 16-bit, on the 256-padded Newton-Schulz buffers."""
    def pad(v):
        return (v + 255) // 256 * 256
    return sum(2 * pad(min(a, b)) ** 2 + 4 * pad(min(a, b)) * pad(max(a, b)) for a, b in shapes)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, indices):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", ",".join(str(i) for i in indices)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons, power = [], [], set(), []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def committed_traffic(kernel_file, workload, prec):
    """DRAM bytes of one APPLY pass over the set (the dominant kernel) from a
    committed ncu summary, or None when the kernel source changed since the
    counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    key = f"ns_apply/{workload}/{prec}"
    if key not in d:
        return None
    src = os.path.join(ROOT, "pretraining_optimizer_b200", "csrc", kernel_file)
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    if d[key].get("source_sha256") != digest:
        return None
    return d[key]["dram_bytes_per_pass"]


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank float over all ranks (device timings are reported as
    the slowest rank's).  NCCL reduces on the rank's GPU, gloo on the CPU."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    if dist.get_backend() == "nccl":
        dev = torch.device("cuda", torch.cuda.current_device())
    else:
        dev = torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, max_ms: float) -> float:
    """Steps per second of the whole job: every rank ran `steps` steps of its
    own replica within the slowest rank's `max_ms`."""
    return world * steps / (max_ms / 1000.0)


# ------------------------------------------------------------------ oracle arm
# NS FLOPs of the oracle's timed sample: one Qwen3-1.7B layer (about 6 s of
# fp64 NumPy on 16 host cores); a set of larger matrices samples fewer.
CPU_SAMPLE_FLOPS = 2.5e12


def cpu_sample(shapes, ns_steps):
    """Indices of the leading matrices of the set (at most 7, one Qwen3 layer)
    whose Newton-Schulz work stays within CPU_SAMPLE_FLOPS; at least one."""
    idx = [0]
    for i in range(1, min(7, len(shapes))):
        if ns_flops(shapes[:i + 1], ns_steps) > CPU_SAMPLE_FLOPS:
            break
        idx.append(i)
    return idx


def oracle_sample_rate(shapes, wl, sample_idx, steps=1):
    """Time the oracle (as it stands, fp64) on a sample of the set for `steps`
    steps; return (steps/s scaled to the whole set, seconds, sample FLOPs share)."""
    import numpy as np
    import oracle
    W0 = {i: wl.weight(i) for i in sample_idx}
    Gs = {(t, i): wl.grad(t, i) for t in range(steps) for i in sample_idx}
    M = {i: np.zeros_like(W0[i], dtype=np.float64) for i in sample_idx}
    W = {i: W0[i].astype(np.float64) for i in sample_idx}
    R = {i: oracle.radius(W0[i]) for i in sample_idx}
    t0 = time.perf_counter()
    for t in range(steps):
        for i in sample_idx:
            W[i], M[i], _, _ = oracle.muonh_step(W[i], M[i], Gs[(t, i)], wl.lrs[t % len(wl.lrs)], R[i],
                                                 wl.beta, wl.nesterov, wl.ns_steps, wl.ns_coeffs)
    dt = time.perf_counter() - t0
    share = ns_flops([shapes[i] for i in sample_idx], wl.ns_steps) / ns_flops(shapes, wl.ns_steps)
    return steps * share / dt, dt, share


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((d.get("num_threads", 1) for d in threadpool_info()), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def bench_config(args, wl, shapes, world):
    """The workload description both arms report."""
    return {"workload": args.workload, "matrices": len(shapes), "params": sum(a * b for a, b in shapes),
            "ns_steps": wl.ns_steps, "ns_precision": args.ns_precision, "state": "fp32 W, M, G",
            "lr": "workload schedule", "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"{world} independent replica(s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl, shapes = workload_desc(args.workload)
    layer0 = list(range(min(7, len(shapes))))
    times, shares = [], []
    for k in range(args.warmup + args.steps):
        idx = [layer0[k % len(layer0)]]           # one matrix of layer 0 per step, in rotation
        _, dt, share = oracle_sample_rate(shapes, wl, idx)
        if k >= args.warmup:
            times.append(dt)
            shares.append(share)
    # each sampled step stands for share of a full step: full-step time = dt / share
    full_step_s = sum(times) / sum(shares)
    value = 1.0 / full_step_s
    cores = blas_threads()
    sample = (f"one layer-0 matrix per step in rotation ({len(layer0)} matrices), fp64 NumPy oracle, "
              f"time scaled to the whole {len(shapes)}-matrix set by Newton-Schulz FLOP share")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * full_step_s,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(args, wl, shapes, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def time_launches(fn, stream, warmup=3, reps=10):
    """Average device time (ms) of fn() over `reps` launches after `warmup`."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_aux(dev, stream, hbm_peak, matrix_params):
    """The two auxiliary kernels of the recipe on the 1.7B model's own sizes,
    each timed alone (burst HBM peak): the AdamW step over the parameters
    outside the matrix set, and the average of six bf16 checkpoints of the
    whole model.  Inputs far exceed L2."""
    import torch
    import synth
    from pretraining_optimizer_b200 import adamw_step, average
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    group = synth.qwen3_adamw_group(2048)
    p = [torch.randn(n, generator=gen, device=dev) * 0.02 for _, n in group]
    m = [torch.zeros_like(x) for x in p]
    v = [torch.zeros_like(x) for x in p]
    g = [torch.randn(x.shape, generator=gen, device=dev) * 1e-3 for x in p]
    n_adam = sum(n for _, n in group)
    adam_ms = time_launches(lambda: adamw_step(p, m, v, g, 1, 1e-3, 0.9, 0.95, 1e-8, 0.1), stream)
    adam_gbps = 28 * n_adam / (adam_ms / 1000.0) / 1e9          # read p, m, v, g; write p, m, v
    del p, m, v, g
    total = n_adam + matrix_params
    ckpts = [torch.randn(total, generator=gen, device=dev, dtype=torch.bfloat16) for _ in range(6)]
    out = torch.empty(total, device=dev, dtype=torch.bfloat16)
    avg_ms = time_launches(lambda: average(ckpts, out=out), stream, reps=5)
    avg_gbps = 14 * total / (avg_ms / 1000.0) / 1e9             # read 6 x 2 B, write 2 B
    del ckpts, out
    torch.cuda.empty_cache()
    return {
        "adamw_step": {"elements": n_adam, "tensors": len(group), "launches": -(-len(group) // 32),
                       "ms": adam_ms, "gbps": adam_gbps, "frac": adam_gbps / hbm_peak,
                       "bytes_per_elem": 28},
        "average": {"elements": total, "checkpoints": 6, "dtype": "bf16 -> bf16", "ms": avg_ms,
                    "gbps": avg_gbps, "frac": avg_gbps / hbm_peak, "bytes_per_elem": 14},
        "peak": "hbm_gbs (burst copy)",
    }


def run_ours(args):
    import torch
    import torch.distributed as dist

    from pretraining_optimizer_b200 import MuonH

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl, shapes = workload_desc(args.workload)
    n = len(shapes)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + rank)
    W = [torch.randn(s, generator=gen, device=dev) * 0.02 for s in shapes]
    M = [torch.zeros_like(w) for w in W]
    G = [torch.randn(s, generator=gen, device=dev) * 1e-3 for s in shapes]
    opt = MuonH(W, M, beta=wl.beta, nesterov=wl.nesterov, ns_steps=wl.ns_steps, ns_coeffs=wl.ns_coeffs,
                ns_precision=args.ns_precision)
    lrs = wl.lrs
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for k in range(args.warmup):
        opt.step(G, lrs[k % len(lrs)])
    torch.cuda.synchronize()
    launches_per_step = opt.last_launch_count()
    opt.phase_times()          # clear any record

    # ---------------- timed region (device events on the launching stream)
    opt.enable_timing(True)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(range(world)) if rank == 0 else None
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        opt.step(G, lrs[k % len(lrs)])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    opt.enable_timing(False)
    ms = t_start.elapsed_time(t_end)
    phases = opt.phase_times()
    opt.device_status()
    ms = max_over_ranks(ms, world)
    ms_per_step = ms / args.steps
    value = whole_job_rate(world, args.steps, ms)

    # ---------------- end to end through the public API, host buffers
    e2e = None
    if not args.no_e2e:
        # gradients as views of one contiguous arena (a training framework's
        # gradient buffer), host side in pinned memory: one copy per step
        sizes = [a * b for a, b in shapes]
        offs = [0]
        for sz in sizes:
            offs.append(offs[-1] + (sz + 63) // 64 * 64)   # 256-byte aligned views

        def views(flat):
            return [flat[o:o + sz].view(s) for o, sz, s in zip(offs, sizes, shapes)]

        host_flat = torch.empty(offs[-1], dtype=torch.float32, pin_memory=True)
        for h, g in zip(views(host_flat), G):
            h.copy_(g)
        stats_dev = torch.empty(n * 6, dtype=torch.int32, device=dev)
        stats_host = torch.empty(n * 6, dtype=torch.int32, pin_memory=True)
        e2e_steps = max(1, min(args.steps, 10))
        # two device gradient arenas: the upload of step k+1's gradients (copy
        # stream) overlaps step k; each step waits for its own upload
        copy = torch.cuda.Stream(device=dev)
        dev_flat = [torch.empty(offs[-1], dtype=torch.float32, device=dev) for _ in range(2)]
        gbuf = [views(f) for f in dev_flat]
        ready = [torch.cuda.Event(), torch.cuda.Event()]
        free = [torch.cuda.Event(), torch.cuda.Event()]

        def upload(b):
            with torch.cuda.stream(copy):
                dev_flat[b].copy_(host_flat, non_blocking=True)
                ready[b].record(copy)

        upload(0)
        opt.step(gbuf[0], lrs[0])      # warm the arena's gradient maps and pages
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy.wait_event(e0)
        upload(0)
        for k in range(e2e_steps):
            b = k & 1
            if k + 1 < e2e_steps:
                if k >= 1:
                    copy.wait_event(free[b ^ 1])   # step k-1 is done with the other buffer
                upload(b ^ 1)
            stream.wait_event(ready[b])
            opt.step(gbuf[b], lrs[k % len(lrs)], stats=stats_dev)
            free[b].record(stream)
            stats_host.copy_(stats_dev, non_blocking=True)
            stream.synchronize()                  # the caller reads the step's stats
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        h2d = 4 * offs[-1]
        e2e = {"value": whole_job_rate(world, e2e_steps, e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": 24 * n, "steps": e2e_steps,
               "pipeline": "gradient upload of step k+1 (pinned host -> device, copy stream) overlaps step k"}
        del host_flat, gbuf, dev_flat

    # ---------------- rooflines from the live per-kernel events
    peaks, peak_src = load_peaks()
    elems = sum(a * b for a, b in shapes)
    kernels = {}
    for name, (tms, cnt) in phases.items():
        if cnt == 0:
            continue
        # a phase may take more than one launch a step (wide and tall tiles)
        entry = {"ms_per_step": tms / args.steps, "launches_per_step": cnt / args.steps,
                 "ms_per_launch": tms / cnt, "share": tms / sum(v[0] for v in phases.values())}
        if name in KERNEL_BYTES:
            entry["gbps"] = KERNEL_BYTES[name] * elems / (tms / args.steps / 1000.0) / 1e9
        kernels[name] = entry
    # APPLY FLOPs of the timed region over the APPLY launches' summed device time
    apply_ms, apply_n = phases["ns_apply"]
    ap_flops = apply_flops(shapes) * wl.ns_steps * args.steps
    achieved = ap_flops / (apply_ms / 1000.0) / 1e12
    peak_t = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    roofline = {"bound": "tensor", "kernel": "ns_apply", "achieved": achieved, "peak": peak_t,
                "unit": "TFLOP/s", "frac": achieved / peak_t,
                "traffic": committed_traffic("muonh_ns_gemm.cu", args.workload, args.ns_precision),
                "per": "one APPLY pass over the set (5 a step; one launch per matrix group)",
                "algorithmic_bytes": apply_bytes(shapes),
                "peak_source": f"bf16_tflops_sustained ({peak_src}); fp16 operands run at the bf16 rate"}
    ns_ms = sum(phases[k][0] for k in ("ns_gram", "ns_square", "ns_apply")) / args.steps
    ew_ms = sum(phases[k][0] for k in ELEMENTWISE) / args.steps
    summary = {
        "ns_tflops_dense": ns_flops(shapes, wl.ns_steps) / (ns_ms / 1000.0) / 1e12,
        "ns_tflops_executed": ns_flops_executed(shapes, wl.ns_steps, args.ns_precision) / (ns_ms / 1000.0) / 1e12,
        "ns_ms_per_step": ns_ms,
        "elementwise_ms_per_step": ew_ms,
        "elementwise_gbps_algorithmic": ALGO_BYTES_PER_ELEM * elems / (ew_ms / 1000.0) / 1e9,
        "hbm_peak_gbps": peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
    }

    # ---------------- auxiliary kernels (rank 0 of a single-GPU run; not part of the step)
    aux = None
    if rank == 0 and world == 1 and not args.no_aux and args.workload == "qwen3_1.7b":
        aux = measure_aux(dev, stream, peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), elems)

    # ---------------- CPU baseline: the oracle on the leading matrices, rank 0, N = 1
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = cpu_sample(shapes, wl.ns_steps)
        rate, dt, share = oracle_sample_rate(shapes, wl, sample)
        cpu = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"the leading {len(sample)} of {n} matrices"
                         f"{' (layer 0)' if args.workload.startswith('qwen3') else ''}, {share:.4f} of the NS "
                         f"FLOPs, one fp64 step ({dt:.1f} s), scaled to the whole set"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f16" if args.ns_precision == "fp16" else
                ("bf16" if args.ns_precision == "bf16" else "f32"),
                "data": "synthetic",
                "config": bench_config(args, wl, shapes, world),
                "roofline": roofline, "summary": summary, "kernels": kernels, "clocks": clocks,
                "gpu_launches": launches_per_step * args.steps, "e2e": e2e, "cpu_baseline": cpu,
                "aux_kernels": aux}
        print(json.dumps(line), flush=True)
    opt.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
