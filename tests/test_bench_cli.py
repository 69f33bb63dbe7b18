"""bench.py's host-side logic on CPU: --gpus N starts N ranks, the reference
arm prints one line from rank 0, and the roofline arithmetic follows the
stated algorithmic byte, flop and exponential counts."""
import json
import os
import subprocess
import sys

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
    """Stands in for the oracle with fixed part times (seconds)."""

    def __init__(self, clock):
        self.clock = clock

    def _tick(self, dt):
        self.clock[0] += dt

    def rpcholesky(self, K, beta, r, seed, eps):
        self._tick(2.0)
        return {"F": None, "S": None, "rank": None}

    def value_range(self, V):
        self._tick(0.5)
        return None, None

    def weights(self, F, S, rank, V):
        self._tick(1.0)
        return None, None

    def gather(self, K, S, rank):
        return None

    def attend(self, *a, rows=None):
        self._tick(0.25)


def test_oracle_extrapolation(monkeypatch):
    """A sampled oracle call is scaled part by part: the select by the summed
    per-step cost to the rank, weights and attend by rank / steps, the attend
    rows by m / rows, the value range not at all."""
    w = workloads.CONFIGS["c4c_long128k"]
    clock = [0.0]
    monkeypatch.setattr(bench.time, "perf_counter", lambda: clock[0])
    rows, steps = bench.oracle_plan(w)
    est, det = bench.oracle_call(_FakeOracle(clock), w, {"K": None, "V": None, "Q": None}, rows, steps)
    s, r, n, d = 64, w.r, w.n, w.d
    sel = (r * d + r * (r - 1) / 2) / (s * d + s * (s - 1) / 2)
    assert det["select_scale"] == pytest.approx(sel)
    assert est == pytest.approx(2.0 * sel + 0.5 + 1.0 * r / s + 0.25 * (w.m / 256) * (r / s))
    # with the device's ranks (here half the instances stop at 256)
    ranks = [512] * 4 + [256] * 4
    clock[0] = 0.0
    est2, det2 = bench.oracle_call(_FakeOracle(clock), w, {"K": None, "V": None, "Q": None}, rows, steps, ranks)
    work = lambda k: k * d + k * (k - 1) / 2
    assert det2["select_scale"] == pytest.approx((work(512) + work(256)) / 2 / work(64))
    assert det2["weights_scale"] == pytest.approx(384 / 64)
