"""The two select kernels -- the per-thread cp.async kernel (the default) and
the bulk-copy kernel (where its shape rules allow) -- against the fp64 oracle
and against each other, and the bulk kernel's bounded-wait path.

- Pivots drawn by either kernel agree with the oracle's own draws step by
  step until a near-tie; on the device's pivots (fixed-pivot mode, the oracle
  following the device's stopping step) every factor column is within 2e-4
  of the oracle's, relative to the column's largest entry.
- On the same fixed pivots the two kernels' factors agree to 2e-4 and stop at
  the same step.
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
def test_both_kernels_match_the_oracle(orc, w, G):
    dev, ex = workloads.make(w)
    K = dev["K"].cuda()
    wc.set_select_cluster(G)
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    for kernel, expect in ((2, (2,)), (1, (1,)), (0, (1, 3, 4)), (4, (1, 4))):
        S, F, rank, K_S, used = _run(K, w, kernel)
        assert used in expect
        if w.name == "kres_g4" and kernel == 4:
            assert used == 4  # resident bf16 keys, d = 64: tensor-core key pass
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


def test_tensor_core_key_pass_recentred(orc):
    """Resident bf16 keys with recentring: the tensor-core key pass splits
    k_s - kbar into three bf16 parts; pivots follow the oracle's draws on
    K - mean(K) and the factor matches the oracle on the device's pivots."""
    w = gc.case("tck_recentre", "walk", 4, 3136, 64, 64, 96, "bf16")
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    wc.set_select_kernel(4)
    O, S, rank = wc.forward_ex(d["Q"], d["K"], d["V"], w.beta, w.r, w.pivot_seed, EPS, recenter=True)
    assert wc.last_select_kernel() == 4
    S, rank = S.cpu().numpy(), rank.cpu().numpy().reshape(w.BH)
    Kc = ex["K"] - ex["K"].mean(axis=1, keepdims=True)
    res = orc.rpcholesky(Kc, w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    gc.pivots_agree_until_tie(S, res["S"], res["margin"], rank, res["rank"])
    fx = orc.wildcat_forward_binned(ex["Q"], ex["K"], ex["V"], w.beta, w.r, 1, eps=0.0, S_fixed=S,
                                    recenter=True)
    lo, hi = orc.value_range(ex["V"])
    assert gc.r12(O.cpu().numpy(), fx[0], lo, hi) <= gc.TOL_R12["bf16"]


@pytest.mark.parametrize("w,G", SHAPES[:5], ids=[w.name for w, _ in SHAPES[:5]])
def test_kernels_agree_on_fixed_pivots(orc, w, G):
    dev, ex = workloads.make(w)
    K = dev["K"].cuda()
    wc.set_select_cluster(G)
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    S_fixed = torch.from_numpy(own["S"]).cuda()
    _, F_a, rank_a, _, used_a = _run(K, w, 2, S_fixed)
    _, F_b, rank_b, _, used_b = _run(K, w, 1, S_fixed)
    _, F_c, rank_c, _, used_c = _run(K, w, 4, S_fixed)
    assert (used_a, used_b) == (2, 1) and used_c in (1, 4)
    assert np.array_equal(rank_a, rank_b) and np.array_equal(rank_c, rank_b)
    assert gc.column_rel_err(F_a, F_b.astype(np.float64), rank_a) < 2e-4
    assert gc.column_rel_err(F_c, F_b.astype(np.float64), rank_c) < 2e-4


def test_recentred_keys_bulk_kernel(orc):
    """The bulk kernel's recentring hook: a forward with recenter on draws
    the pivots the oracle draws on K - mean(K)."""
    w = gc.case("recentre", "iid", 2, 2048, 64, 64, 48, "bf16")
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    wc.set_select_kernel(2)
    O, S, rank = wc.forward_ex(d["Q"], d["K"], d["V"], w.beta, w.r, w.pivot_seed, EPS, recenter=True)
    assert wc.last_select_kernel() == 2
    S, rank = S.cpu().numpy(), rank.cpu().numpy().reshape(w.BH)
    _, S_o, rank_o = orc.wildcat_forward_binned(ex["Q"], ex["K"], ex["V"], w.beta, w.r, 1,
                                                seed=w.pivot_seed, eps=EPS, recenter=True)
    res = orc.rpcholesky(ex["K"] - ex["K"].mean(axis=1, keepdims=True), w.beta, w.r,
                         seed=w.pivot_seed, eps=EPS)
    assert np.array_equal(S_o, res["S"])
    gc.pivots_agree_until_tie(S, res["S"], res["margin"], rank, res["rank"])


def test_bulk_select_bounded_wait_reports_timeout_and_recovers():
    """The test hook makes every CTA's warp 0 wait 1 ms, after step 1, on a
    barrier phase nothing completes.  The expiry is recorded in the device
    status word, the abort reaches every CTA of the cluster with the chunk
    sums, all stop after two steps, and the next call is clean."""
    w = gc.case("sel_timeout", "iid", 3, 4096, 64, 64, 32, "bf16")
    dev, _ = workloads.make(w)
    K = dev["K"].cuda()
    wc.set_select_cluster(4)
    wc.set_select_kernel(2)
    assert wc.device_status() == 0
    wc.force_select_timeout(1_000_000)
    try:
        S, F, rank, _ = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
        assert wc.last_select_kernel() == 2
        assert wc.device_status() == 5
        assert torch.all(rank == 2)
        assert torch.all(S[:, 2:] == -1)
    finally:
        wc.force_select_timeout(0)
    S, F, rank, _ = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
    assert wc.device_status() == 0
    assert torch.all(rank == w.r)


GS_SHAPES = [
    gc.case("gs_bh2_d128", "iid", 2, 16384, 64, 128, 64, "bf16"),
    gc.case("gs_bh8_d128", "iid", 8, 16384, 64, 128, 48, "bf16"),
    gc.case("gs_ragged_f32", "iid", 3, 20000, 64, 64, 50, "f32"),
    gc.case("gs_walk_trunc", "walk", 4, 16384, 64, 128, 300, "bf16"),
]


@pytest.mark.parametrize("w", GS_SHAPES, ids=lambda w: w.name)
def test_global_sync_form_matches_the_oracle(orc, w):
    """The cp.async kernel in global-sync form (CTAs of an instance meet at a
    counter barrier in the workspace): same checks as above, and the same
    factorisation as the cluster form on the same pivots."""
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
