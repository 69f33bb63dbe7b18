#!/usr/bin/env python
"""Benchmark of the WildCat forward (select -> weights -> attend) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, same metric

One step = one wildcat_forward call over the whole workload (all instances)
with inputs resident in device memory.  The default workload is the largest
single-GPU one: the long-context sweep at n = m = 131072 (8 heads, d = 128,
r = 512, bf16).  Each step is bracketed by its own CUDA events on the
launching stream; a 256 MiB device write flushes the L2 cache between steps,
outside the events.  With N > 1 (one rank per GPU, started by torchrun or,
when --gpus N is given without it, by this script re-launching itself under
torch.distributed.run) every rank runs its own copy of the workload (weak
scaling; instances are independent, so there is no collective on the data
path) and the reported time is the maximum over ranks.

Printed (rank 0): one JSON line with the metric, the device-timed value,
an end-to-end value through wildcat_forward_host (with --nbins > 1,
wildcat_forward_ex_host; pinned host buffers, copies inside the timed region), per-stage times with each stage's
roofline fraction (select and weights against HBM bandwidth, attend against
the bf16 tensor peak), the forward-level roofline (sum over stages of
max(bytes / HBM, MMA flops / tensor peak, exps / MUFU rate) against the
measured step time), the roofline of the dominant kernel, sampled SM clocks,
and the oracle timed on the host cores as a CPU baseline.  Where the oracle
cannot afford a whole call it runs a stated sample and extrapolates each
part from two sample sizes, a fixed cost plus a cost that grows with the
size (the line says so): when m > 4096 the attend on 1024 and 4096 seeded
rows per head, and, when one instance's select is large (the 65536- and
131072-token workloads), the select and weights on the first 32 and 64
pivot steps of every instance (step i of the select costs n (d + i)).
"""
from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "WildCat fwd calls/s & effective m*n attention entries/s on 1 B200; % roofline"
FLUSH_BYTES = 256 << 20
EPS = 1e-6
ORACLE_FULL_ROWS_MAX = 4096   # above this m the oracle's attend runs on sampled rows
ORACLE_SAMPLE_ROWS = 256
MUFU_EX2_PER_CLK_SM = 16      # exponentials per clock per SM (SFU), nominal
SM_COUNT = 148


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["wildcat", "reference"], default="wildcat")
    p.add_argument("--workload", default="c4c_long128k")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="minimum CPU time of the baseline leg when whole calls are cheap")
    p.add_argument("--nbins", type=int, default=1,
                   help="divide-and-conquer bins (1 = the unbinned method)")
    p.add_argument("--select-cluster", type=int, default=0,
                   help="CTAs per instance in the select (0 = automatic; a fixed size keeps 512-thread CTAs)")
    p.add_argument("--weights-inverse", action="store_true",
                   help="also time the inverse-maintenance weights route on the selected pivots")
    p.add_argument("--select-phase-steps", type=int, default=0,
                   help="select steps per launch (0 = automatic: 64 for r >= 512; < 0 = one launch)")
    p.add_argument("--select-kernel", type=int, choices=[0, 1, 3], default=0,
                   help="0 = automatic, 1 = clusters, 3 = global sync where it applies")
    return p.parse_args()


def relaunch_if_needed(args):
    """--gpus N > 1 outside torchrun: start N ranks under torch.distributed.run
    (this script again, same arguments) and return their exit status.
    Inside torchrun the world size must equal --gpus.  Returns None when this
    process should run the benchmark itself."""
    world = os.environ.get("WORLD_SIZE")
    if world is None:
        if args.gpus <= 1:
            return None
        with socket.socket() as s:
            s.bind(("127.0.0.1", 0))
            port = s.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
               "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
        return subprocess.call(cmd)
    if int(world) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        return 2
    return None


def workload_config(w, extra=None):
    cfg = {"workload": f"{w.name}: BH={w.BH} (B={w.B}, H={w.H}), n={w.n}, m={w.m}, d={w.d}, "
                       f"r={w.r}, {w.dtype} inputs, {w.dist} keys",
           "BH": w.BH, "n": w.n, "m": w.m, "d": w.d, "r": w.r, "input_dtype": w.dtype,
           "accumulate": "f32", "beta": w.beta, "distribution": w.dist}
    if extra:
        cfg.update(extra)
    return cfg


def in_bytes(w):
    return 2 if w.dtype == "bf16" else 4


def select_bytes(w, ranks):
    """Algorithmic bytes of one RPCholesky select: per step i the key pass
    (n d b_K), the factor prefix read (4 n i), the new column write (4 n) and
    the residual read + write (8 n)."""
    bk = in_bytes(w)
    total = 0
    for rr in ranks:
        rr = int(rr)
        total += rr * w.n * (w.d * bk + 12) + 2 * w.n * rr * (rr - 1)
    return total


def weights_bytes(w, ranks):
    """Algorithmic bytes of the weights stage: the factor's r' rows read once
    (4 r' n) and V read once (n d b_V)."""
    return sum(4 * int(rr) * w.n + w.n * w.d * in_bytes(w) for rr in ranks)


def attend_work(w, ranks):
    """(MMA flops, exponentials, HBM bytes) of the attend: GEMM1 Q K_S^T and
    GEMM2 P V_S at 2 m r' d flops each, m r' exponentials, Q read and the
    float32 output written."""
    flops = sum(4.0 * w.m * int(rr) * w.d for rr in ranks)
    exps = sum(float(w.m) * int(rr) for rr in ranks)
    nbytes = w.BH * w.m * w.d * (in_bytes(w) + 4)
    return flops, exps, nbytes


def read_peaks():
    """HBM GB/s and bf16 TFLOP/s (burst, sustained) measured on this machine, else
    the stated fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


SELECT_KERNELS = {
    # last_select_kernel() code -> kernel name
    1: "rpc_select_kernel",
    3: "rpc_select_kernel (global sync)",
}


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


# ---------------------------------------------------------------------------
# the fp64 CPU oracle, as it stands (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

ORACLE_FULL_SELECT_WORK = 5e9   # per-instance select work n (r d + r^2 / 2) above which the oracle is sampled
ORACLE_SAMPLE_STEPS = 64
ORACLE_TIMING_ROWS = 4096       # rows of the larger sample that times a sampled attend


def oracle_plan(w):
    """What the oracle runs per call: (rows, steps).  rows: every query row, or
    256 seeded rows per head when m is large; steps: every pivot step, or the
    first 64 of every instance when one instance's select is large (c4b, c4c:
    tens of seconds of fp64 per instance)."""
    import workloads

    rows = None if w.m <= ORACLE_FULL_ROWS_MAX else workloads.sample_rows(w, ORACLE_SAMPLE_ROWS)
    steps = None
    if w.n * (w.r * w.d + w.r * w.r / 2) > ORACLE_FULL_SELECT_WORK:
        steps = min(w.r, ORACLE_SAMPLE_STEPS)
    return rows, steps


def _select_work(w, k):
    # the oracle's pivot step i costs n (d + i) multiply-adds (kernel column and factor prefix)
    return w.n * (k * w.d + k * (k - 1) / 2.0)


def _timed(fn):
    t0 = time.perf_counter()
    out = fn()
    return out, time.perf_counter() - t0


def oracle_call(orc, w, ex, rows, steps=None, ranks=None):
    """One oracle forward (select, value range, weights, gather, attend),
    timed per part.  rows: the attend's query rows (None = all); steps: pivot
    steps run (None = all r).  Returns (seconds for a whole call, detail).
    With sampled steps the select and weights also run on half the steps, and
    a fixed part plus a part growing with the steps (the select's step i
    costs n (d + i); the weights grow with the coreset size) are fitted and
    taken to each instance's rank (`ranks`, default r); the value range is
    timed in full.  A sampled attend runs with a coreset of the full size r (the
    first r keys when the steps were sampled: its cost depends on the sizes
    only) on half of `rows` and on all of them, and is extrapolated to m rows
    by the fitted cost: a fixed part (the query-norm pass over all m rows,
    the setup) plus a per-row part."""
    s = w.r if steps is None else steps
    sel, t_sel = _timed(lambda: orc.rpcholesky(ex["K"], w.beta, s, seed=w.pivot_seed, eps=EPS))
    (vmin, vmax), t_rng = _timed(lambda: orc.value_range(ex["V"]))
    (VS, wv), t_wt = _timed(lambda: orc.weights(sel["F"], sel["S"], sel["rank"], ex["V"]))
    if steps is not None:
        # the same on half the steps: a fixed part (the prologue's pass over
        # the keys, setup) and a part that grows with the steps are fitted
        s2 = max(1, s // 2)
        sel2, t_sel2 = _timed(lambda: orc.rpcholesky(ex["K"], w.beta, s2, seed=w.pivot_seed, eps=EPS))
        _, t_wt2 = _timed(lambda: orc.weights(sel2["F"], sel2["S"], sel2["rank"], ex["V"]))
    KS, rank_att = orc.gather(ex["K"], sel["S"], sel["rank"]), sel["rank"]
    if steps is not None:
        # a coreset of the full size for timing the attend (its values do not change its cost)
        full = np.tile(np.arange(w.r, dtype=np.int32), (w.BH, 1))
        rank_att = np.full(w.BH, w.r, dtype=np.int32)
        KS = orc.gather(ex["K"], full, rank_att)
        VS = np.zeros((w.BH, w.r, w.d))
        wv = np.ones((w.BH, w.r))

    def att(rs):
        return _timed(lambda: orc.attend(ex["Q"], KS, VS, wv, rank_att, vmin, vmax, w.beta, rows=rs))[1]

    if rows is None:
        t_att = att(None)
        att_det = {"attend_s": t_att, "attend_rows": w.m}
    else:
        import workloads

        # two seeded row samples large enough that the per-row cost shows
        # above the fixed part (rows cost the same)
        na, nb = min(w.m, ORACLE_TIMING_ROWS // 4), min(w.m, ORACLE_TIMING_ROWS)
        t1, t2 = att(workloads.sample_rows(w, na)), att(workloads.sample_rows(w, nb))
        per_row = max(0.0, (t2 - t1) / (nb - na))
        fixed = max(0.0, t1 - per_row * na)
        t_att = fixed + per_row * w.m
        att_det = {"attend_rows_timed": [na, nb], "attend_s_timed": [t1, t2], "attend_fixed_s": fixed,
                   "attend_per_row_s": per_row, "attend_extrapolated_s": t_att}
    if steps is None:
        est_sel, est_wt = t_sel, t_wt
        det = {"select_s": t_sel, "weights_s": t_wt}
    else:
        rk = [w.r] * w.BH if ranks is None else [max(1, int(x)) for x in ranks]
        # select: fixed + b * work(steps), work = n (steps d + steps (steps - 1) / 2)
        b_sel = max(0.0, (t_sel - t_sel2) / (_select_work(w, s) - _select_work(w, s2)))
        a_sel = max(0.0, t_sel - b_sel * _select_work(w, s))
        est_sel = a_sel + b_sel * statistics.mean(_select_work(w, k) for k in rk)
        # weights: fixed + b * coreset size
        b_wt = max(0.0, (t_wt - t_wt2) / (s - s2))
        a_wt = max(0.0, t_wt - b_wt * s)
        est_wt = a_wt + b_wt * statistics.mean(rk)
        det = {"select_steps_timed": [s2, s], "select_s_timed": [t_sel2, t_sel], "select_extrapolated_s": est_sel,
               "weights_s_timed": [t_wt2, t_wt], "weights_extrapolated_s": est_wt}
    est = est_sel + t_rng + est_wt + t_att
    det["value_range_s"] = t_rng
    det.update(att_det)
    return est, det


def oracle_sample_text(w, rows, reps=None, steps=None):
    if rows is None and steps is None:
        return (f"{reps} whole wildcat_forward calls of the workload ({w.BH} instances), fp64, "
                "OpenMP over instances")
    parts = []
    if steps is None:
        parts.append(f"select and weights in full on all {w.BH} instances")
    else:
        parts.append(f"select on the first {steps // 2} and {steps} of the r = {w.r} pivot steps of all {w.BH} "
                     f"instances, extrapolated to each instance's rank by the fitted fixed + per-step cost "
                     f"(step i costs n (d + i)); weights on those pivots, extrapolated linearly in the coreset "
                     f"size; value range in full")
    if rows is None:
        parts.append("attend on every query row")
    else:
        parts.append(f"attend with an r-row coreset on {ORACLE_TIMING_ROWS // 4} and {ORACLE_TIMING_ROWS} "
                     f"seeded query rows per head, extrapolated to m = {w.m} rows by the fitted fixed + "
                     "per-row cost")
    return "; ".join(parts) + "; fp64, OpenMP over instances"


def oracle_binned_call(orc, w, ex, nb):
    """One oracle binned forward (nb bins): whole when m <= 4096, else the
    whole call on 1024 and on 4096 seeded query rows per head, extrapolated to
    m rows by the fitted fixed (select, weights, query pass) + per-row cost."""
    def call(rows):
        t0 = time.perf_counter()
        orc.wildcat_forward_binned(ex["Q"], ex["K"], ex["V"], w.beta, w.r, nb, seed=w.pivot_seed, eps=EPS,
                                   rows=rows)
        return time.perf_counter() - t0

    if w.m <= ORACLE_FULL_ROWS_MAX:
        t = call(None)
        return t, {"binned_call_s": t}
    import workloads

    na, nbr = ORACLE_TIMING_ROWS // 4, ORACLE_TIMING_ROWS
    t1, t2 = call(workloads.sample_rows(w, na)), call(workloads.sample_rows(w, nbr))
    per_row = max(0.0, (t2 - t1) / (nbr - na))
    fixed = max(0.0, t1 - per_row * na)
    est = fixed + per_row * w.m
    return est, {"rows_timed": [na, nbr], "s_timed": [t1, t2], "fixed_s": fixed, "per_row_s": per_row}


def oracle_step(orc, w, ex, nb=1, ranks=None):
    """The oracle's time for one call of the bench's workload: (seconds,
    detail, whole, sample text).  whole: a whole call was timed as is."""
    if nb > 1:
        est, det = oracle_binned_call(orc, w, ex, nb)
        whole = w.m <= ORACLE_FULL_ROWS_MAX
        text = (f"one whole binned wildcat_forward ({nb} bins, {w.BH} instances)" if whole else
                f"binned wildcat_forward ({nb} bins, {w.BH} instances) on {ORACLE_TIMING_ROWS // 4} and "
                f"{ORACLE_TIMING_ROWS} seeded query rows per head, extrapolated to m = {w.m} rows by the fitted "
                "fixed + per-row cost") + "; fp64, OpenMP over instances"
        return est, det, whole, text
    rows, steps = oracle_plan(w)
    if rows is None and steps is None:
        t0 = time.perf_counter()
        orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
        return time.perf_counter() - t0, None, True, (f"one whole wildcat_forward call of the workload "
                                                      f"({w.BH} instances), fp64")
    est, det = oracle_call(orc, w, ex, rows, steps, ranks)
    return est, det, False, oracle_sample_text(w, rows, steps=steps)


def cpu_baseline(w, ex, seconds, ranks=None, nb=1):
    """The fp64 oracle, as it stands, on the host cores: whole calls repeated
    for `seconds`, or one sampled call (oracle_plan, oracle_binned_call) when a
    call is large; `ranks`: the effective rank of every instance from the
    device run, for the extrapolation of sampled pivot steps; nb: bins."""
    import oracle

    orc = oracle.get()
    T = orc.num_threads()
    used = {"select_and_weights": min(w.BH * nb, T), "attend": T}  # OpenMP over instances / over query rows
    est, det, whole, text = oracle_step(orc, w, ex, nb, ranks)
    if not whole:
        return {"value": 1.0 / est, "unit": "calls/s", "cores": T, "threads_used": used, "kind": "oracle",
                "partial": True, "sample": text, "seconds_per_call": est, "detail": det}
    reps, el = 1, est
    while el < seconds:
        el += oracle_step(orc, w, ex, nb, ranks)[0]
        reps += 1
    return {"value": reps / el, "unit": "calls/s", "cores": T, "threads_used": used, "kind": "oracle",
            "partial": False, "sample": f"{reps} calls: {text}"}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on the same workload and metric
    (rank 0 only; other ranks exit at once)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import oracle
    import workloads

    w = workloads.CONFIGS[args.workload]
    _, ex = workloads.make(w)
    orc = oracle.get()
    nb = max(1, args.nbins)
    for _ in range(max(args.warmup, 3)):
        oracle_step(orc, w, ex, nb)
    secs, det, whole, text = [], None, True, ""
    for _ in range(args.steps):
        est, det, whole, text = oracle_step(orc, w, ex, nb)
        secs.append(est)
    total = sum(secs)
    value = args.steps / total
    T = orc.num_threads()
    cpu = {"value": value, "unit": "calls/s", "cores": T, "kind": "oracle",
           "threads_used": {"select_and_weights": min(w.BH * nb, T), "attend": T},
           "partial": not whole, "sample": ("one step per call; " + text)}
    if det is not None:
        cpu["detail_last_step"] = det
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "calls/s",
           "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
           "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(w, {"l2": "n/a (host)", "nbins": nb}),
           "entries_per_s": value * w.BH * w.m * w.n,
           "cpu_baseline": cpu,
           "e2e": {"value": value, "unit": "calls/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------------------
# rooflines
# ---------------------------------------------------------------------------

def count_library_launches(fn):
    """Kernels that one call of fn launches (fn calls only this library, so
    every kernel in the trace is one of its own), from the CUDA activity
    trace of torch.profiler; copies and memsets are not counted.  None if the
    profiler is unavailable.  Run outside the timed region."""
    import torch

    try:
        from torch.autograd import DeviceType
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == DeviceType.CUDA
                 and not e.name.startswith(("Memcpy", "Memset"))]
        return len(names)
    except Exception:
        return None


def stage_rooflines(w, ranks_sel, ranks_att, stage_ms, peaks, nbins=1):
    """Per-stage achieved rates, their roofline fractions and the forward-level
    roofline time.  ranks_sel: effective ranks of the select problems (per bin
    when binned); ranks_att: coreset size per instance seen by the attend."""
    wb = w.scaled(n=w.n // nbins) if nbins > 1 else w
    bw = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops_sustained"] * 1e12
    mufu = MUFU_EX2_PER_CLK_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e6
    sb = select_bytes(wb, ranks_sel)
    wtb = weights_bytes(wb, ranks_sel)
    af, ae, ab = attend_work(w, ranks_att)
    ms = {k: statistics.mean(v) for k, v in stage_ms.items()}
    out = {
        "select": {"ms": ms["select"], "bytes": sb, "achieved_gbs": sb / (ms["select"] / 1e3) / 1e9,
                   "bound": "hbm", "frac": sb / (ms["select"] / 1e3) / bw,
                   "roofline_ms": 1e3 * sb / bw},
        "weights": {"ms": ms["weights"], "bytes": wtb,
                    "achieved_gbs": wtb / (ms["weights"] / 1e3) / 1e9, "bound": "hbm",
                    "frac": wtb / (ms["weights"] / 1e3) / bw, "roofline_ms": 1e3 * wtb / bw},
        "attend": {"ms": ms["attend"], "mma_flops": af, "exps": ae, "bytes": ab,
                   "achieved_tflops": af / (ms["attend"] / 1e3) / 1e12, "bound": "tensor",
                   "frac": af / (ms["attend"] / 1e3) / tc,
                   "roofline_ms": 1e3 * max(af / tc, ae / mufu, ab / bw),
                   "limits_ms": {"tensor": 1e3 * af / tc, "mufu": 1e3 * ae / mufu, "hbm": 1e3 * ab / bw}},
    }
    total = sum(v["roofline_ms"] for v in out.values())
    peaks_used = {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops_sustained": peaks["bf16_tflops_sustained"],
                  "mufu_ex2_per_s": mufu, "source": peaks["source"] + " (MUFU: 16/clk/SM x 148 x max clock)"}
    return out, total, peaks_used


def main():
    args = parse()
    rc = relaunch_if_needed(args)
    if rc is not None:
        return rc
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
    ranks_att = plan.rank.reshape(w.BH, -1).sum(dim=1).cpu().tolist()
    sel_kind = wc.last_select_kernel()
    sel_cluster = wc.last_select_cluster()
    sel_threads = wc.last_select_threads()
    sel_launches = wc.last_select_phases()
    launches = count_library_launches(lambda: plan.run(Q, K, V, w.beta, w.pivot_seed, EPS))

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
        peak64 = SM_COUNT * 64 * 2 * 1.965e9 / 1e12
        ach = (zflops + invflops) / (ms_inv / 1e3) / 1e12
        inv = {"ms": ms_inv, "fp64_flops_per_call": zflops + invflops, "achieved_tflops": ach,
               "peak_tflops": peak64, "frac": ach / peak64, "bound": "alu",
               "peak_source": "fp64 unit count: 148 SMs x 64 FMA/clk x 2 x 1.965 GHz"}

    # ---- end to end through wildcat_forward_host / wildcat_forward_ex_host (host buffers) ----
    e2e = None
    if not args.no_e2e:
        if nb == 1:
            hp = wc.HostForwardPlan(w.BH, w.m, w.n, w.d, w.r, w.dtype)
            api = "wildcat_forward_host (pinned host buffers)"
        else:
            hp = wc.HostForwardExPlan(w.BH, w.m, w.n, w.d, w.r, w.dtype, nbins=nb)
            api = f"wildcat_forward_ex_host with nbins = {nb} (pinned host buffers)"
        pinned = {k: v.pin_memory() for k, v in dev.items()}
        O_host = torch.empty((w.BH, w.m, w.d), dtype=torch.float32).pin_memory()
        S_host = torch.empty((w.BH, w.r), dtype=torch.int32).pin_memory()
        r_host = torch.empty((w.BH, nb) if nb > 1 else (w.BH,), dtype=torch.int32).pin_memory()
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
        eb = in_bytes(w)
        e2e = {"value": world * args.steps / (e_tot / 1e3), "unit": "calls/s",
               "h2d_bytes_per_step": eb * w.BH * (w.m + 2 * w.n) * w.d,
               "d2h_bytes_per_step": 4 * w.BH * w.m * w.d + 4 * w.BH * w.r + 4 * w.BH * nb,
               "api": api}
        del hp

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(w, ex, args.cpu_seconds, ranks=plan.rank.cpu().tolist() if nb == 1 else None, nb=nb)

    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    value = world * args.steps / (total_ms / 1e3)
    peaks = read_peaks()
    stages, roof_ms, peaks_used = stage_rooflines(w, ranks, ranks_att, stage_ms, peaks, nb)
    sel = stages["select"]
    ms_per_step = total_ms / args.steps
    # the select's factor of one rank's batch (bins: the largest instance group in flight is all of it)
    factor_mb = 4.0 * w.BH * (w.r // nb) * (w.n // nb) * nb / 1e6
    out = {
        "metric": METRIC, "value": value, "unit": "calls/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": workload_config(w0, {"l2": "flushed between steps (256 MiB device write)",
                                       "parallelism": f"instances per rank x {world} ranks",
                                       "nbins": nb,
                                       "select_kernel": SELECT_KERNELS.get(sel_kind, str(sel_kind)),
                                       "select_cluster_ctas": sel_cluster,
                                       "select_cta_threads": sel_threads,
                                       "select_launches": sel_launches}),
        "entries_per_s": value * w.BH * w.m * w.n,
        "stages_ms": {k: v["ms"] for k, v in stages.items()},
        "stages": stages,
        "forward_roofline": {"roofline_ms": roof_ms, "measured_ms": ms_per_step,
                             "pct": 100.0 * roof_ms / ms_per_step,
                             "rule": "sum over stages of max(bytes / HBM, MMA flops / bf16 sustained, "
                                     "exps / MUFU)", "peaks": peaks_used},
        "roofline": {"kernel": SELECT_KERNELS.get(sel_kind, str(sel_kind)), "bound": "hbm",
                     "achieved": sel["achieved_gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": sel["frac"], "peak_source": f"{peaks['source']} hbm_gbs",
                     "traffic": None,
                     "algorithmic_bytes_per_call": sel["bytes"], "call_ms": sel["ms"],
                     "launches_per_call": sel_launches,
                     "bytes_model": ("streaming model: the factor prefix and keys re-read every step; "
                                     + ("the factor (%.0f MB) fits in the 126 MB L2, so part of these bytes "
                                        "are L2 hits and the kernel is bound by its per-step latency, not "
                                        "DRAM" % (factor_mb,) if factor_mb < 126 else
                                        "the factor (%.0f MB) exceeds the L2, so these are DRAM bytes" % (factor_mb,)))},
        "gpu_launches": None if launches is None else launches * args.steps,
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
