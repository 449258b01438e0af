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
NS_PHASES = ("ns_gram", "ns_square", "ns_product", "ns_apply")
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
    ap.add_argument("--groups", type=int, default=0, choices=[0, 1, 2, 3],
                    help="matrix groups of the step (0: the library's automatic choice)")
    ap.add_argument("--ns-form", default="auto", choices=["auto", "y", "gram"],
                    help="Newton-Schulz evaluation: Gram-space runs where they save FLOPs (auto), "
                         "Y-space everywhere, or Gram-space wherever fp16 allows")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-aux", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the side records (elementwise alone, bf16, Qwen3-0.6B, shape sweep)")
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


def committed_traffic(kernel_file, phase, workload, prec):
    """DRAM bytes of one step's launches of the dominant kernel phase from a
    committed ncu summary, or None when the kernel source changed since the
    counters were taken (or none were taken for this phase and workload)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    key = f"{phase}/{workload}/{prec}"
    if key not in d:
        return None
    src = os.path.join(ROOT, "pretraining_optimizer_b200", "csrc", kernel_file)
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    if d[key].get("source_sha256") != digest:
        return None
    return d[key]["dram_bytes_per_step"]


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
    steps, its Newton-Schulz products and its elementwise work (momentum,
    norms, the Eq. (1) projection) apart, each called in the order of
    oracle.muonh_step.  The whole-set step time is each part's time scaled by
    its own share of the set (NS FLOPs, elements).  Returns (steps/s of the
    whole set, seconds timed, NS FLOP share, element share)."""
    import numpy as np
    import oracle
    W0 = {i: wl.weight(i) for i in sample_idx}
    Gs = {(t, i): wl.grad(t, i) for t in range(steps) for i in sample_idx}
    M = {i: np.zeros_like(W0[i], dtype=np.float64) for i in sample_idx}
    W = {i: W0[i].astype(np.float64) for i in sample_idx}
    R = {i: oracle.radius(W0[i]) for i in sample_idx}
    t_ns = t_ew = 0.0
    for t in range(steps):
        for i in sample_idx:
            t0 = time.perf_counter()
            M[i], X = oracle.momentum_update(M[i], Gs[(t, i)], wl.beta, wl.nesterov)
            float(np.linalg.norm(X))
            t1 = time.perf_counter()
            O = oracle.newton_schulz(X, wl.ns_steps, wl.ns_coeffs)
            t2 = time.perf_counter()
            W[i], _ = oracle.hyperball_update(W[i], O, wl.lrs[t % len(wl.lrs)], R[i])
            t3 = time.perf_counter()
            t_ew += (t1 - t0) + (t3 - t2)
            t_ns += t2 - t1
    ns_share = ns_flops([shapes[i] for i in sample_idx], wl.ns_steps) / ns_flops(shapes, wl.ns_steps)
    el_share = sum(shapes[i][0] * shapes[i][1] for i in sample_idx) / sum(a * b for a, b in shapes)
    full_step_s = (t_ns / ns_share + t_ew / el_share) / steps
    return 1.0 / full_step_s, t_ns + t_ew, ns_share, el_share


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((d.get("num_threads", 1) for d in threadpool_info()), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def bench_config(args, wl, shapes, world):
    """The workload description both arms report."""
    return {"workload": args.workload, "matrices": len(shapes), "params": sum(a * b for a, b in shapes),
            "ns_steps": wl.ns_steps, "ns_precision": args.ns_precision, "ns_form": args.ns_form,
            "groups": args.groups,
            "state": "fp32 W, M, G",
            "lr": "workload schedule", "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"{world} independent replica(s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl, shapes = workload_desc(args.workload)
    layer0 = list(range(min(7, len(shapes))))
    step_s = []
    for k in range(args.warmup + args.steps):
        idx = [layer0[k % len(layer0)]]           # one matrix of layer 0 per step, in rotation
        rate, _, _, _ = oracle_sample_rate(shapes, wl, idx)
        if k >= args.warmup:
            step_s.append(1.0 / rate)
    full_step_s = sum(step_s) / len(step_s)
    value = 1.0 / full_step_s
    cores = blas_threads()
    sample = (f"one layer-0 matrix per step in rotation ({len(layer0)} matrices), fp64 NumPy oracle on "
              f"{os.cpu_count()} host cores ({cores} BLAS threads); its Newton-Schulz time scaled to the whole "
              f"{len(shapes)}-matrix set by NS FLOP share, its elementwise time by element share")
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


def time_set(shapes, wl, prec, groups, warmup, steps, dev, stream, seed, ns_form="auto"):
    """One context over `shapes` with device-drawn inputs of the workload's
    distributions: `warmup` untimed steps, then `steps` steps bracketed by
    CUDA events on the launching stream with per-kernel timing on.  Returns
    (ms per step, {phase: (ms, launches)} of the timed steps, {phase:
    executed tensor FLOPs per step})."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    W = [torch.randn(s, generator=gen, device=dev) * 0.02 for s in shapes]
    M = [torch.zeros_like(w) for w in W]
    G = [torch.randn(s, generator=gen, device=dev) * 1e-3 for s in shapes]
    opt = MuonH(W, M, beta=wl.beta, nesterov=wl.nesterov, ns_steps=wl.ns_steps, ns_coeffs=wl.ns_coeffs,
                ns_precision=prec, groups=groups, ns_form=ns_form)
    lrs = wl.lrs
    for k in range(warmup):
        opt.step(G, lrs[k % len(lrs)])
    torch.cuda.synchronize()
    opt.phase_times()
    opt.enable_timing(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(steps):
        opt.step(G, lrs[k % len(lrs)])
    e1.record(stream)
    torch.cuda.synchronize()
    opt.enable_timing(False)
    phases = opt.phase_times()
    flops = opt.phase_flops()
    opt.device_status()
    opt.close()
    del W, M, G
    torch.cuda.empty_cache()
    return e0.elapsed_time(e1) / steps, phases, flops


def ns_record(ms, phases, flops, steps, peak_t):
    """Newton-Schulz rates of a timed set: executed TFLOP/s over the GEMM
    phases, and the most time-consuming GEMM phase's TFLOP/s against the
    sustained peak."""
    ns = [k for k in NS_PHASES if phases[k][1] > 0]
    ns_ms = sum(phases[k][0] for k in ns) / steps
    dom = max(ns, key=lambda k: phases[k][0])
    dom_t = flops[dom] / (phases[dom][0] / steps / 1000.0) / 1e12
    return {"steps_per_s": 1000.0 / ms, "ms_per_step": ms, "ns_ms_per_step": ns_ms,
            "ns_tflops_executed": sum(flops[k] for k in ns) / (ns_ms / 1000.0) / 1e12,
            "dominant": dom, "dominant_tflops": dom_t, "dominant_frac": dom_t / peak_t}


def side_records(dev, stream, peaks, args):
    """Measurements beside the headline line, each its own context on fresh
    device inputs (rank 0 of a single-GPU run):
      elementwise_alone  the momentum and projection kernels of the Qwen3-1.7B
                         set, each kind of tile on its own (tall: gate and up;
                         wide: the rest) with the step in one group, so no
                         launch overlaps another; against the burst HBM peak;
      bf16               the Qwen3-1.7B set with bf16 Newton-Schulz operands;
      qwen3_0.6b         the Qwen3-0.6B set (fp16 operands, its WSD schedule);
      sweep              each shape of the roofline sweep in one group: the
                         executed NS TFLOP/s and each elementwise kernel's GB/s."""
    import synth
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    peak_t = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    sampler = ClockSampler([torch_device_index(dev)])
    out = {}
    wl17, shapes17 = workload_desc("qwen3_1.7b")

    def ew(phases, name, elems, per_elem):
        t, cnt = phases[name]
        ms = t / cnt
        gbps = per_elem * elems / ms / 1e6
        return {"ms_per_launch": ms, "launches": cnt, "gbps": gbps, "frac": gbps / hbm}

    alone = {}
    for kind, sub in (("tall", [s for s in shapes17 if s[0] > s[1]]), ("wide", [s for s in shapes17 if s[0] <= s[1]])):
        ms, ph, _ = time_set(sub, wl17, "fp16", 1, 3, 5, dev, stream, seed=11)
        el = sum(a * b for a, b in sub)
        alone[kind] = {"matrices": len(sub), "elements": el,
                       "momentum_norm": ew(ph, "momentum_norm", el, KERNEL_BYTES["momentum_norm"]),
                       "project": ew(ph, "project", el, KERNEL_BYTES["project"])}
    alone["peak"] = "hbm_gbs (burst copy): each launch runs alone"
    out["elementwise_alone"] = alone

    ms, ph, fl = time_set(shapes17, wl17, "bf16", 0, 3, 10, dev, stream, seed=12)
    out["bf16"] = {"workload": "qwen3_1.7b", "ns_precision": "bf16", "ns_form": "y (bf16 runs the Y-space form)",
                   **ns_record(ms, ph, fl, 10, peak_t)}

    ms, ph, fl = time_set(shapes17, wl17, "fp16", 0, 3, 10, dev, stream, seed=15, ns_form="y")
    out["fp16_y_space"] = {"workload": "qwen3_1.7b", "ns_precision": "fp16", "ns_form": "y",
                           **ns_record(ms, ph, fl, 10, peak_t)}

    wl06, shapes06 = workload_desc("qwen3_0.6b")
    ms, ph, fl = time_set(shapes06, wl06, "fp16", 0, 5, 20, dev, stream, seed=13)
    el06 = sum(a * b for a, b in shapes06)
    ew06 = sum(ph[k][0] for k in ELEMENTWISE if k in ph) / 20
    out["qwen3_0.6b"] = {"workload": "qwen3_0.6b", "matrices": len(shapes06), "params": el06,
                         **ns_record(ms, ph, fl, 20, peak_t),
                         "elementwise_gbps_algorithmic": ALGO_BYTES_PER_ELEM * el06 / (ew06 / 1000.0) / 1e9}

    sweep = []
    for r, c in synth.SWEEP_SHAPES:
        wls, shs = workload_desc(f"sweep_{r}x{c}")
        ms, ph, fl = time_set(shs, wls, "fp16", 1, 3, 3, dev, stream, seed=14)
        el = sum(a * b for a, b in shs)
        sweep.append({"shape": [r, c], "matrices": len(shs), **ns_record(ms, ph, fl, 3, peak_t),
                      "momentum_norm_gbps": ew(ph, "momentum_norm", el, KERNEL_BYTES["momentum_norm"])["gbps"],
                      "project_gbps": ew(ph, "project", el, KERNEL_BYTES["project"])["gbps"]})
    out["sweep"] = sweep
    out["side_clocks"] = sampler.stop()
    return out


def torch_device_index(dev):
    return dev.index if dev.index is not None else 0


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
                ns_precision=args.ns_precision, ns_form=args.ns_form, groups=args.groups)
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
        e2e_steps = max(1, args.steps)
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
    # Newton-Schulz rooflines from the FLOPs each phase's tiles execute (the
    # library counts them per launch) over the phase's summed device time;
    # the dominant kernel is the GEMM phase that takes the most time
    flops = opt.phase_flops()
    ns_phases = [k for k in NS_PHASES if phases[k][1] > 0]
    for k in ns_phases:
        kernels[k]["tflops_executed"] = flops[k] / (phases[k][0] / args.steps / 1000.0) / 1e12
    dom = max(ns_phases, key=lambda k: phases[k][0])
    achieved = kernels[dom]["tflops_executed"]
    peak_t = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak_t,
                "unit": "TFLOP/s", "frac": achieved / peak_t,
                "traffic": committed_traffic("muonh_ns_gemm.cu", dom, args.workload, args.ns_precision),
                "per": f"the {dom} launches of one step ({phases[dom][1] // args.steps} a step)",
                "flops_per_step": flops[dom],
                "peak_source": f"bf16_tflops_sustained ({peak_src}); fp16 operands run at the bf16 rate"}
    ns_ms = sum(phases[k][0] for k in ns_phases) / args.steps
    ew_ms = sum(phases[k][0] for k in ELEMENTWISE) / args.steps
    summary = {
        "ns_form": args.ns_form,
        "ns_tflops_method_dense": ns_flops(shapes, wl.ns_steps) / (ns_ms / 1000.0) / 1e12,
        "ns_tflops_executed": sum(flops[k] for k in ns_phases) / (ns_ms / 1000.0) / 1e12,
        "ns_flops_executed_per_step": sum(flops[k] for k in ns_phases),
        "ns_ms_per_step": ns_ms,
        "elementwise_ms_per_step": ew_ms,
        "elementwise_gbps_algorithmic": ALGO_BYTES_PER_ELEM * elems / (ew_ms / 1000.0) / 1e9,
        "hbm_peak_gbps": peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
    }

    # ---------------- auxiliary kernels (rank 0 of a single-GPU run; not part of the step)
    aux = None
    if rank == 0 and world == 1 and not args.no_aux and args.workload == "qwen3_1.7b":
        aux = measure_aux(dev, stream, peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), elems)

    # ---------------- side records (rank 0 of a single-GPU run of the headline set)
    side = {}
    if rank == 0 and world == 1 and not args.no_extra and args.workload == "qwen3_1.7b":
        opt.close()
        opt = None
        del W, M, G
        torch.cuda.empty_cache()
        side = side_records(dev, stream, peaks, args)

    # ---------------- CPU baseline: the oracle on the leading matrices, rank 0, N = 1
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = cpu_sample(shapes, wl.ns_steps)
        rate, dt, share, el_share = oracle_sample_rate(shapes, wl, sample)
        cpu = {"value": rate, "unit": UNIT, "cores": blas_threads(), "nproc": os.cpu_count(), "kind": "oracle",
               "sample": f"one measured fp64 step ({dt:.1f} s) of the leading {len(sample)} of {n} matrices"
                         f"{' (layer 0)' if args.workload.startswith('qwen3') else ''}: {share:.4f} of the NS "
                         f"FLOPs and {el_share:.4f} of the elements; Newton-Schulz and elementwise times "
                         f"scaled to the whole set by their own shares"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f16" if args.ns_precision == "fp16" else
                ("bf16" if args.ns_precision == "bf16" else "f32"),
                "data": "synthetic",
                "config": bench_config(args, wl, shapes, world),
                "roofline": roofline, "summary": summary, "kernels": kernels, "clocks": clocks,
                "gpu_launches": launches_per_step * args.steps, "e2e": e2e, "cpu_baseline": cpu,
                "aux_kernels": aux, **side}
        print(json.dumps(line), flush=True)
    if opt is not None:
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
