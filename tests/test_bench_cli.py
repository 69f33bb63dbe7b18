"""bench.py's host-side logic on CPU: --gpus N starts N ranks, the reference
arm prints one line from rank 0, and the roofline arithmetic follows the
stated algorithmic byte, flop and exponential counts."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def _run(args, env_extra=None):
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=300)


def test_gpus_two_starts_two_ranks():
    p = _run(["--gpus", "2", "--impl", "reference", "--workload", "c0_unit", "--steps", "1",
              "--warmup", "3"])
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2
    assert out["steps"] == 1 and out["warmup"] == 3
    assert out["e2e"]["h2d_bytes_per_step"] == 0


def test_world_size_must_match_gpus():
    p = _run(["--gpus", "2", "--impl", "reference", "--workload", "c0_unit"],
             {"WORLD_SIZE": "1", "RANK": "0", "LOCAL_RANK": "0"})
    assert p.returncode != 0
    assert "WORLD_SIZE" in p.stderr


def test_default_workload_is_the_largest_single_gpu_config():
    args = sys.argv
    try:
        sys.argv = ["bench.py"]
        a = bench.parse()
    finally:
        sys.argv = args
    w = workloads.CONFIGS[a.workload]
    assert a.workload == "c4c_long128k"
    assert w.BH * w.m * w.n == max(c.BH * c.m * c.n for c in workloads.CONFIGS.values())


def test_stage_rooflines_recompute():
    w = workloads.CONFIGS["c4c_long128k"]
    ranks = [512] * w.BH
    peaks = {"hbm_gbs": 6545.3, "bf16_tflops": 1668.5, "bf16_tflops_sustained": 1391.0,
             "sm_max_mhz": 1965.0, "source": "measured"}
    stage_ms = {"select": [100.0], "weights": [2.0], "attend": [0.5]}
    st, roof_ms, _ = bench.stage_rooflines(w, ranks, ranks, stage_ms, peaks)
    # select: sum_b r n (d b_K + 12) + 2 n r (r - 1), the streaming model's bytes
    sb = w.BH * (512 * w.n * (w.d * 2 + 12) + 2 * w.n * 512 * 511)
    assert st["select"]["bytes"] == sb
    assert st["select"]["frac"] == pytest.approx(sb / 0.1 / 6545.3e9)
    # weights: 4 r' n + 2 n d per instance
    wb = w.BH * (4 * 512 * w.n + 2 * w.n * w.d)
    assert st["weights"]["bytes"] == wb
    # attend: 4 m r' d MMA flops, m r' exponentials, Q read + fp32 O written
    af = w.BH * 4.0 * w.m * 512 * w.d
    assert st["attend"]["mma_flops"] == af
    assert st["attend"]["frac"] == pytest.approx(af / 0.5e-3 / 1391e12)
    mufu = 16 * 148 * 1965e6
    att_roof = max(af / 1391e12, w.BH * w.m * 512 / mufu, w.BH * w.m * w.d * 6 / 6545.3e9)
    assert roof_ms == pytest.approx(1e3 * (sb / 6545.3e9 + wb / 6545.3e9 + att_roof))


def test_oracle_sampling_rule():
    assert bench.oracle_plan(workloads.CONFIGS["c1_vit56"]) == (None, None)
    assert bench.oracle_plan(workloads.CONFIGS["c4a_long16k"])[1] is None  # select in full
    rows, steps = bench.oracle_plan(workloads.CONFIGS["c4c_long128k"])
    assert len(rows) == 256 and len(set(rows.tolist())) == 256 and steps == 64


class _FakeOracle:
    """Stands in for the oracle: each part's time is a fixed cost plus a cost
    that grows with its size, so the bench's extrapolation can be checked
    against the exact time of a whole call."""

    def __init__(self, clock, w):
        self.clock, self.w = clock, w

    def sel_time(self, k):
        return 0.3 + 2e-12 * self.w.n * (k * self.w.d + k * (k - 1) / 2)

    def wt_time(self, k):
        return 0.2 + 0.01 * k

    def att_time(self, nrows):
        return 0.05 + 1e-5 * nrows

    def rpcholesky(self, K, beta, r, seed, eps):
        self.clock[0] += self.sel_time(r)
        return {"F": None, "S": np.zeros((self.w.BH, r), np.int32), "rank": np.full(self.w.BH, r, np.int32)}

    def value_range(self, V):
        self.clock[0] += 0.5
        return None, None

    def weights(self, F, S, rank, V):
        self.clock[0] += self.wt_time(S.shape[1])
        return None, None

    def gather(self, K, S, rank):
        return None

    def attend(self, *a, rows=None):
        self.clock[0] += self.att_time(self.w.m if rows is None else len(rows))


def test_oracle_extrapolation(monkeypatch):
    """A sampled oracle call is extrapolated part by part from two sample
    sizes (fixed + growing cost): with part times that follow that model
    exactly, the estimate equals the whole call's time."""
    w = workloads.CONFIGS["c4c_long128k"]
    clock = [0.0]
    monkeypatch.setattr(bench.time, "perf_counter", lambda: clock[0])
    fake = _FakeOracle(clock, w)
    rows, steps = bench.oracle_plan(w)
    est, det = bench.oracle_call(fake, w, {"K": None, "V": None, "Q": None}, rows, steps)
    whole = fake.sel_time(w.r) + 0.5 + fake.wt_time(w.r) + fake.att_time(w.m)
    assert est == pytest.approx(whole, rel=1e-9)
    # with the device's ranks (here half the instances stop at 256)
    ranks = [512] * 4 + [256] * 4
    est2, _ = bench.oracle_call(fake, w, {"K": None, "V": None, "Q": None}, rows, steps, ranks)
    sel = 0.3 + 2e-12 * w.n * ((512 * w.d + 512 * 511 / 2) + (256 * w.d + 256 * 255 / 2)) / 2
    assert est2 == pytest.approx(sel + 0.5 + (0.2 + 0.01 * 384) + fake.att_time(w.m), rel=1e-9)
