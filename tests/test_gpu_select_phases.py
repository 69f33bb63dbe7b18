"""Phased select: the steps of one call run as several launches; between them
the instances still going keep their residual diagonal in the workspace and
continue in a global-sync launch that shares the whole GPU among them.

- On every shape the pivots agree with the oracle's own draws until a
  near-tie, the factor matches the oracle's on the device's pivots (2e-4 of
  each column's largest entry), K_S is the exact gather, and the same call in
  one launch draws the same pivots.
- Instances that truncate inside a phase stop there; the rest pause at the
  phase end and resume (ragged last phase included).
- A bounded barrier wait that runs out inside a resumed launch is reported,
  every instance stops two steps into that launch, and the next call is clean.
"""
import math

import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

EPS = 1e-6

# (case, steps per launch, select kernel of the first launch: 0 automatic, 1 clusters, 3 global sync)
PHASE_SHAPES = [
    (gc.case("ph_walk_trunc", "walk", 8, 8192, 64, 128, 400, "bf16"), 64, 0),   # truncation inside phases
    (gc.case("ph_iid_gs", "iid", 4, 16384, 64, 128, 64, "bf16"), 24, 3),        # 24 + 24 + 16 steps
    (gc.case("ph_iid_cluster", "iid", 6, 8192, 64, 64, 48, "bf16"), 16, 1),     # first launch on clusters
    (gc.case("ph_f32", "iid", 3, 4096, 64, 64, 40, "f32"), 8, 0),               # float32 keys, five launches
]


@pytest.fixture(autouse=True)
def _restore_knobs():
    yield
    wc.set_select_kernel(0)
    wc.set_select_phase_steps(0)
    wc.force_select_timeout(0)


def _select(K, w, steps):
    wc.set_select_phase_steps(steps)
    S, F, rank, K_S = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
    torch.cuda.synchronize()
    return S.cpu().numpy(), F.cpu().numpy(), rank.cpu().numpy(), K_S, wc.last_select_phases()


@pytest.mark.parametrize("w,steps,kernel", PHASE_SHAPES, ids=[w.name for w, _, _ in PHASE_SHAPES])
def test_phases_match_the_oracle(orc, w, steps, kernel):
    dev, ex = workloads.make(w)
    K = dev["K"].cuda()
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    wc.set_select_kernel(kernel)
    S, F, rank, K_S, launches = _select(K, w, steps)
    assert launches == math.ceil(w.r / steps)
    if kernel:
        assert wc.last_select_kernel() == kernel
    gc.pivots_agree_until_tie(S, own["S"], own["margin"], rank, own["rank"], F, own["F"], EPS)
    for b in range(w.BH):
        rr = rank[b]
        assert rr >= 1 and len(set(S[b, :rr].tolist())) == rr and np.all(S[b, rr:] == -1)
        assert np.all(F[b, rr:] == 0)
    fx = orc.rpcholesky(ex["K"], w.beta, w.r, eps=0.0, S_fixed=S)
    assert np.array_equal(fx["rank"], rank)
    assert gc.column_rel_err(F, fx["F"], rank) < 2e-4
    KS_ref = orc.gather(ex["K"], S, rank)
    assert np.array_equal(K_S.float().cpu().numpy().astype(np.float64), KS_ref)
    # one launch: the same pivots until a float32 near-tie
    S1, F1, rank1, _, launches1 = _select(K, w, -1)
    assert launches1 == 1
    gc.pivots_agree_until_tie(S1, own["S"], own["margin"], rank1, own["rank"], F1, own["F"], EPS)
    assert wc.device_status() == 0


def test_phases_cover_paused_and_truncated_instances(orc):
    """With a larger eps the instances stop at different steps, some inside the
    first launch and some in later ones; every rank equals the oracle's on the
    device's pivots."""
    w = gc.case("ph_eps", "walk", 12, 8192, 64, 128, 256, "bf16")
    eps = 1e-3
    dev, ex = workloads.make(w)
    K = dev["K"].cuda()
    wc.set_select_phase_steps(32)
    S, F, rank, K_S = wc.select(K, w.beta, w.r, w.pivot_seed, eps)
    torch.cuda.synchronize()
    assert wc.last_select_phases() == 8
    S, F, rank = S.cpu().numpy(), F.cpu().numpy(), rank.cpu().numpy()
    assert rank.min() < rank.max()
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=eps)
    gc.pivots_agree_until_tie(S, own["S"], own["margin"], rank, own["rank"], F, own["F"], eps)
    fx = orc.rpcholesky(ex["K"], w.beta, w.r, eps=eps, S_fixed=S)
    assert np.array_equal(fx["rank"], rank)
    assert gc.column_rel_err(F, fx["F"], rank) < 2e-4
    assert wc.device_status() == 0


def test_resumed_phase_barrier_timeout_reports_and_recovers():
    """The first launch runs on clusters (no counter barrier); in the second,
    CTA 0 of every instance skips its third counter barrier, the bounded waits
    end (1 ms), the timeout is recorded, every instance stops after two steps
    of that launch, and the next call is clean."""
    w = gc.case("ph_timeout", "iid", 2, 16384, 64, 128, 48, "bf16")
    dev, _ = workloads.make(w)
    K = dev["K"].cuda()
    wc.set_select_kernel(1)
    wc.set_select_phase_steps(16)
    assert wc.device_status() == 0
    wc.force_select_timeout(1_000_000)
    try:
        S, F, rank, _ = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
        assert wc.last_select_phases() == 3
        assert wc.device_status() == 5
        assert torch.all(rank == 16 + 2)
    finally:
        wc.force_select_timeout(0)
    S, F, rank, _ = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
    assert wc.device_status() == 0
    assert torch.all(rank == w.r)
