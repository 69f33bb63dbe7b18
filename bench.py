#!/usr/bin/env python
"""Benchmark of the WildCat forward (select -> weights -> attend) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, same metric

One step = one wildcat_forward call over the whole workload (all instances)
with inputs resident in device memory.  Each step is bracketed by its own
CUDA events on the launching stream; a 256 MiB device write flushes the L2
cache between steps, outside the events.  With N > 1 (torchrun, one rank per
GPU) every rank runs its own copy of the workload (weak scaling; instances
are independent, so there is no collective on the data path) and the
reported time is the maximum over ranks.

Printed (rank 0): one JSON line with the metric, the device-timed value,
an end-to-end value through wildcat_forward_host (pinned host buffers,
copies inside the timed region), a per-stage breakdown, the roofline of the
dominant kernel (the RPCholesky select), sampled SM clocks, and the oracle
timed on the host cores as a CPU baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "WildCat fwd calls/s & effective m*n attention entries/s on 1 B200; % roofline"
FLUSH_BYTES = 256 << 20
EPS = 1e-6


def launches_per_forward(w, select_launches=1):
    """Kernels one wildcat_forward launches: select 1 (or one per phase of a
    long coreset), weights 5 (range partial and finalize, F^T(V,1),
    pivot-block gather, solve), attend 3 on CUDA cores (norm partials, shift,
    attend) or 4 on the tensor-core path (plus the hi/lo split of [V_S|w])."""
    tc = w.dtype == "bf16" and w.d in (64, 128)
    return select_launches + 5 + (4 if tc else 3)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["wildcat", "reference"], default="wildcat")
    p.add_argument("--workload", default="c1_vit56")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--nbins", type=int, default=1,
                   help="divide-and-conquer bins (1 = the unbinned method)")
    p.add_argument("--select-cluster", type=int, default=0,
                   help="CTAs per instance in the select (0 = automatic; a fixed size keeps 512-thread CTAs)")
    p.add_argument("--weights-inverse", action="store_true",
                   help="also time the inverse-maintenance weights route on the selected pivots")
    p.add_argument("--select-phase-steps", type=int, default=0,
                   help="select steps per launch (0 = automatic: 64 for r >= 512; < 0 = one launch)")
    p.add_argument("--select-kernel", type=int, choices=[0, 1, 2, 3, 4], default=0,
                   help="0 = automatic (the cp.async kernel), 1 = cp.async, 2 = bulk-copy where it applies")
    return p.parse_args()


def workload_config(w, extra=None):
    cfg = {"workload": f"{w.name}: BH={w.BH} (B={w.B}, H={w.H}), n={w.n}, m={w.m}, d={w.d}, "
                       f"r={w.r}, {w.dtype} inputs, {w.dist} keys",
           "BH": w.BH, "n": w.n, "m": w.m, "d": w.d, "r": w.r, "input_dtype": w.dtype,
           "beta": w.beta, "distribution": w.dist}
    if extra:
        cfg.update(extra)
    return cfg


def select_bytes(w, ranks):
    """Algorithmic bytes of one RPCholesky select launch: per step i the key
    pass (n d b_K), the factor prefix read (4 n i), the new column write (4 n)
    and the residual read + write (8 n)."""
    bk = 2 if w.dtype == "bf16" else 4
    total = 0
    for rr in ranks:
        rr = int(rr)
        total += rr * w.n * (w.d * bk + 12) + 2 * w.n * rr * (rr - 1)
    return total


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


SELECT_KERNELS = {
    # last_select_kernel() code -> (kernel name, profile prefix, source files)
    1: ("rpc_select_kernel", "rpc_select", ("select.cu", "common.cuh", "philox.cuh")),
    2: ("rpc_select_bulk_kernel", "rpc_select_bulk",
        ("select_bulk.cu", "common.cuh", "philox.cuh", "tc_common.cuh")),
    3: ("rpc_select_kernel (global sync)", "rpc_select_gs", ("select.cu", "common.cuh", "philox.cuh")),
    4: ("rpc_select_kernel (tensor-core key pass)", "rpc_select",
        ("select.cu", "common.cuh", "philox.cuh", "tc_common.cuh")),
}


def kernel_source_hash(kind=1):
    h = hashlib.sha256()
    for name in SELECT_KERNELS[kind][2]:
        with open(os.path.join(ROOT, "nystr_coreset_approximate_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name, kind=1, launches=1):
    """DRAM bytes of one select call (the sum over its launches when it runs
    in phases) from a committed ncu summary, if it was taken on the current
    kernel source with the same number of launches; else None."""
    path = os.path.join(ROOT, "profiles", f"{SELECT_KERNELS[kind][1]}_{workload_name}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_call = re.search(r"dram_bytes_per_call:\s*([0-9.eE+]+)", text)
    m_tr = m_call or re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_n = re.search(r"select_launches:\s*([0-9]+)", text)
    if not m_hash or not m_tr or m_hash.group(1) != kernel_source_hash(kind):
        return None
    if (int(m_n.group(1)) if m_n else 1) != launches:
        return None
    return float(m_tr.group(1))


class ClockSampler:
    """nvidia-smi samples during the timed region (sm clock, reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[4:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for _, _, r in rows for k in range(4) if r[k + 1] == "Active"})
        return {"sm_mhz": statistics.median(s for s, _, _ in rows),
                "sm_max_mhz": max(m for _, m, _ in rows), "reasons": reasons,
                "samples": len(rows)}


def cpu_baseline(w, ex, seconds):
    """The fp64 oracle, as it stands, on the host cores over the whole workload."""
    import oracle

    orc = oracle.get()
    reps, t0 = 0, time.perf_counter()
    while True:
        orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": reps / el, "unit": "calls/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{reps} full wildcat_forward calls of the whole workload "
                      f"({w.BH} instances) in {el:.1f} s, fp64, OpenMP over instances"}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on the same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import workloads

    w = workloads.CONFIGS[args.workload]
    _, ex = workloads.make(w)
    orc = oracle.get()
    for _ in range(args.warmup):
        orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps / total
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "calls/s",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(w, {"l2": "n/a (host)"}),
           "entries_per_s": value * w.BH * w.m * w.n,
           "cpu_baseline": {"value": value, "unit": "calls/s", "cores": orc.num_threads(),
                            "kind": "oracle",
                            "sample": f"the whole workload per step ({w.BH} instances), fp64"},
           "e2e": {"value": value, "unit": "calls/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import nystr_coreset_approximate_b200 as wc
    import workloads
    from nystr_coreset_approximate_b200 import sharding

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    wc.set_select_kernel(args.select_kernel)
    wc.set_select_cluster(args.select_cluster)
    wc.set_select_phase_steps(args.select_phase_steps)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    w0 = workloads.CONFIGS[args.workload]
    w = w0.scaled(seed=w0.seed + 1000 * rank)  # each rank its own batch of instances
    dev, ex = workloads.make(w)
    Q, K, V = (dev[k].cuda() for k in ("Q", "K", "V"))
    nb = max(1, args.nbins)
    if nb > 1:
        plan = wc.BinnedForwardPlan(w.BH, w.m, w.n, w.d, w.r, nb, w.dtype)
    else:
        plan = wc.ForwardPlan(w.BH, w.m, w.n, w.d, w.r, w.dtype)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- warm-up ----
    for _ in range(max(args.warmup, 3)):
        plan.run(Q, K, V, w.beta, w.pivot_seed, EPS)
    torch.cuda.synchronize()
    ranks = plan.rank.reshape(-1).cpu().tolist()  # per instance (per bin when binned)
    sel_kind = wc.last_select_kernel()
    sel_cluster = wc.last_select_cluster()
    sel_threads = wc.last_select_threads()
    sel_launches = wc.last_select_phases()

    # ---- timed forward: K steps, own events per step, L2 flushed in between ----
    clocks = ClockSampler(local)
    clocks.start()
    # each timed forward also records stage markers on its own stream (after the
    # select's launches, after the weights'), so the stage split and the select
    # kernel's time come from the timed calls themselves
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    after_sel = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    after_wt = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for ev in after_sel + after_wt:
        ev.record()  # creates the handle the library records into
    torch.cuda.synchronize()
    barrier()
    for k in range(args.steps):
        flush.zero_()
        wc.set_stage_events(after_sel[k], after_wt[k])
        starts[k].record()
        plan.run(Q, K, V, w.beta, w.pivot_seed, EPS)
        ends[k].record()
    wc.set_stage_events(None, None)
    barrier()
    clk = clocks.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sharding.max_over_ranks(sum(step_ms), device="cuda")

    # ---- per-stage split of the timed forwards (binned: the attend stage also
    #      holds the union of the bins' coresets) ----
    stage_ms = {"select": [s.elapsed_time(e) for s, e in zip(starts, after_sel)],
                "weights": [s.elapsed_time(e) for s, e in zip(after_sel, after_wt)],
                "attend": [s.elapsed_time(e) for s, e in zip(after_wt, ends)]}
    inv = None
    if args.weights_inverse and nb == 1:
        # the inverse route (fp64) on the same pivots; ALU-bound by its Z contraction
        inv_ms = []
        for k in range(args.steps + 2):
            flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            wc.weights_inverse(K, plan.S, plan.rank, V, w.beta)
            a1.record()
            torch.cuda.synchronize()
            if k >= 2:
                inv_ms.append(a0.elapsed_time(a1))
        rks = plan.rank.cpu().tolist()
        zflops = sum(4.0 * rr * w.n * (w.d + 1) for rr in rks)       # dot products + accumulation, fp64
        invflops = sum(4.0 * rr ** 3 / 3.0 + 2.0 * rr * rr * (w.d + 1) for rr in rks)
        ms_inv = statistics.mean(inv_ms)
        peak64 = 148 * 64 * 2 * 1.965e9 / 1e12
        ach = (zflops + invflops) / (ms_inv / 1e3) / 1e12
        inv = {"ms": ms_inv, "fp64_flops_per_call": zflops + invflops, "achieved_tflops": ach,
               "peak_tflops": peak64, "frac": ach / peak64, "bound": "alu",
               "peak_source": "fp64 unit count: 148 SMs x 64 FMA/clk x 2 x 1.965 GHz"}
    sel_ms = statistics.mean(stage_ms["select"])

    # ---- end to end through wildcat_forward_host (host buffers) ----
    e2e = None
    if not args.no_e2e and nb == 1:
        hp = wc.HostForwardPlan(w.BH, w.m, w.n, w.d, w.r, w.dtype)
        pinned = {k: v.pin_memory() for k, v in dev.items()}
        O_host = torch.empty((w.BH, w.m, w.d), dtype=torch.float32).pin_memory()
        S_host = torch.empty((w.BH, w.r), dtype=torch.int32).pin_memory()
        r_host = torch.empty((w.BH,), dtype=torch.int32).pin_memory()
        for _ in range(2):
            hp.run(pinned["Q"], pinned["K"], pinned["V"], O_host, w.beta, w.pivot_seed, EPS,
                   S_host, r_host)
        barrier()
        e_ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            hp.run(pinned["Q"], pinned["K"], pinned["V"], O_host, w.beta, w.pivot_seed, EPS,
                   S_host, r_host)
            b.record()
            b.synchronize()
            e_ms.append(a.elapsed_time(b))
        e_tot = sharding.max_over_ranks(sum(e_ms), device="cuda")
        eb = 2 if w.dtype == "bf16" else 4
        e2e = {"value": world * args.steps / (e_tot / 1e3), "unit": "calls/s",
               "h2d_bytes_per_step": eb * w.BH * (w.m + 2 * w.n) * w.d,
               "d2h_bytes_per_step": 4 * w.BH * w.m * w.d + 4 * w.BH * w.r + 4 * w.BH,
               "api": "wildcat_forward_host (pinned host buffers)"}
        del hp

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(w, ex, args.cpu_seconds)

    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    value = world * args.steps / (total_ms / 1e3)
    peak, peak_kind = read_peaks()
    nbytes = select_bytes(w.scaled(n=w.n // nb), ranks)
    achieved = nbytes / (sel_ms / 1e3) / 1e9
    traffic = recorded_traffic(w0.name if nb == 1 else f"{w0.name}_bins{nb}", sel_kind, sel_launches)
    out = {
        "metric": METRIC, "value": value, "unit": "calls/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(w0, {"l2": "flushed between steps (256 MiB device write)",
                                       "parallelism": f"instances per rank x {world} ranks",
                                       "nbins": nb,
                                       "select_kernel": SELECT_KERNELS[sel_kind][0],
                                       "select_cluster_ctas": sel_cluster,
                                       "select_cta_threads": sel_threads,
                                       "select_launches": sel_launches}),
        "entries_per_s": value * w.BH * w.m * w.n,
        "stages_ms": {k: statistics.mean(v) for k, v in stage_ms.items()},
        "roofline": {"kernel": SELECT_KERNELS[sel_kind][0], "bound": "hbm", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} hbm_gbs", "traffic": traffic,
                     "algorithmic_bytes_per_launch": nbytes, "launch_ms": sel_ms,
                     "launches_per_select": sel_launches},
        "gpu_launches": (launches_per_forward(w, sel_launches) + (1 if nb > 1 else 0)) * args.steps,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "effective_rank_mean": sum(ranks) / len(ranks),
    }
    if inv is not None:
        out["weights_inverse"] = inv
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
