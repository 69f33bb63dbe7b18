"""The select kernel's two forms -- clusters (distributed shared memory, the
hardware cluster barrier) and global sync (a cooperative grid meeting at a
bounded counter barrier in the workspace) -- against the fp64 oracle and
against each other, and the global-sync barrier's bounded-wait path.

- Pivots drawn by either form agree with the oracle's own draws step by
  step until a near-tie; on the device's pivots (fixed-pivot mode, the oracle
  following the device's stopping step) every factor column is within 2e-4
  of the oracle's, relative to the column's largest entry.
- A bounded wait that runs out (the test hook) is reported through the
  device status word, every instance stops at the same step, and the next
  call is clean.
"""
import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

EPS = 1e-6

# (case, cluster size or 0 = automatic); the comment names the code path
SHAPES = [
    (gc.case("kres_g4", "mixture16", 4, 3136, 3136, 64, 128, "bf16"), 0),    # resident keys, 4 CTAs
    (gc.case("stream_g1", "iid", 3, 4096, 64, 64, 200, "bf16"), 0),          # streamed keys, 1 CTA, contiguous stages
    (gc.case("stream_g16", "iid", 2, 16384, 64, 128, 96, "bf16"), 0),        # 16-CTA clusters
    (gc.case("rows8192", "iid", 2, 32768, 64, 128, 40, "bf16"), 4),          # 8192 rows per CTA, 4 quads per thread
    (gc.case("f32_d32", "iid", 3, 1000, 64, 32, 50, "f32"), 0),              # float32, two column groups
    (gc.case("tiny_full", "iid", 2, 12, 12, 32, 12, "f32"), 0),              # 12 rows, 16 column groups, full rank
    (gc.case("ragged_g8", "iid", 2, 5000, 64, 64, 64, "bf16"), 8),           # last CTA shorter than the rest
    (gc.case("walk_trunc", "walk", 2, 8192, 64, 128, 400, "bf16"), 0),       # early truncation
]


@pytest.fixture(autouse=True)
def _restore_knobs():
    yield
    wc.set_select_kernel(0)
    wc.set_select_cluster(0)
    wc.force_select_timeout(0)


def _run(K, w, kernel, S_fixed=None):
    wc.set_select_kernel(kernel)
    if S_fixed is None:
        S, F, rank, K_S = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
    else:
        S, F, rank, K_S = wc.select_fixed(K, w.beta, S_fixed, EPS)
    torch.cuda.synchronize()
    used = wc.last_select_kernel()
    return S.cpu().numpy(), F.cpu().numpy(), rank.cpu().numpy(), K_S, used


@pytest.mark.parametrize("w,G", SHAPES, ids=[w.name for w, _ in SHAPES])
def test_cluster_form_matches_the_oracle(orc, w, G):
    dev, ex = workloads.make(w)
    K = dev["K"].cuda()
    wc.set_select_cluster(G)
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    for kernel, expect in ((1, (1,)), (0, (1, 3))):
        S, F, rank, K_S, used = _run(K, w, kernel)
        assert used in expect
        if w.name == "kres_g4" and kernel == 0 and G == 0:
            # automatic: two 256-thread CTAs per SM, 8 per instance
            assert wc.last_select_threads() == 256 and wc.last_select_cluster() == 8
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
    assert wc.device_status() == 0


GS_SHAPES = [
    gc.case("gs_bh2_d128", "iid", 2, 16384, 64, 128, 64, "bf16"),
    gc.case("gs_bh8_d128", "iid", 8, 16384, 64, 128, 48, "bf16"),
    gc.case("gs_ragged_f32", "iid", 3, 20000, 64, 64, 50, "f32"),
    gc.case("gs_walk_trunc", "walk", 4, 16384, 64, 128, 300, "bf16"),
]


@pytest.mark.parametrize("w", GS_SHAPES, ids=lambda w: w.name)
def test_global_sync_form_matches_the_oracle(orc, w):
    """The global-sync form (CTAs of an instance meet at a counter barrier in
    the workspace): same checks as above, and the cluster form draws the same
    pivots."""
    dev, ex = workloads.make(w)
    K = dev["K"].cuda()
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    S, F, rank, K_S, used = _run(K, w, 3)
    assert used == 3 and wc.last_select_cluster() > 16 // 2
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
    # the cluster form draws the same pivots until a float32 near-tie
    S1, F1, rank1, _, used1 = _run(K, w, 1)
    assert used1 == 1
    gc.pivots_agree_until_tie(S1, own["S"], own["margin"], rank1, own["rank"], F1, own["F"], EPS)
    assert wc.device_status() == 0


def test_global_sync_forward_matches_staged_calls(orc):
    """wildcat_forward picks the global-sync form for few long instances; its
    output equals the staged calls (select through the workspace) bit for bit."""
    w = gc.case("gs_forward", "iid", 2, 16384, 256, 128, 64, "bf16")
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O_f, S_f, rank_f = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, w.pivot_seed, EPS)
    assert wc.last_select_kernel() == 3
    S, F, rank, K_S = wc.select(d["K"], w.beta, w.r, w.pivot_seed, EPS)
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, d["V"])
    O = wc.attend(d["Q"], K_S, rank, w.beta, V_S, wv, vmin, vmax)
    assert torch.equal(S_f, S) and torch.equal(rank_f, rank) and torch.equal(O_f, O)
    assert wc.device_status() == 0


def test_global_sync_barrier_timeout_reports_and_recovers():
    """The test hook keeps CTA 0 of every instance from arriving at the third
    counter barrier; every CTA's bounded wait ends (1 ms), the timeout is
    recorded, all stop after one step, and the next call is clean."""
    w = gc.case("gs_timeout", "iid", 2, 16384, 64, 128, 32, "bf16")
    dev, _ = workloads.make(w)
    K = dev["K"].cuda()
    wc.set_select_kernel(3)
    assert wc.device_status() == 0
    wc.force_select_timeout(1_000_000)
    try:
        S, F, rank, _ = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
        assert wc.last_select_kernel() == 3
        assert wc.device_status() == 5
        assert torch.all(rank == 1)
    finally:
        wc.force_select_timeout(0)
    S, F, rank, _ = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
    assert wc.last_select_kernel() == 3
    assert wc.device_status() == 0
    assert torch.all(rank == w.r)
