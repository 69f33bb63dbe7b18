"""Device path vs the fp64 oracle, element by element, at sizes the oracle
finishes in seconds that span several tiles, several CTAs per instance and
ragged tails (n not a multiple of 4 or of the search chunk, r not a
multiple of the GEMM tile, m not a multiple of the query tile).

Every call goes through the C ABI (libwildcat.so) via the thin binding."""
import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

EPS = 1e-6

CASES = [
    gc.case("f32_iid", "iid", 2, 1000, 333, 64, 40, "f32"),
    gc.case("f32_d32_vec1", "iid", 3, 1023, 130, 32, 17, "f32"),
    gc.case("f32_d128", "iid", 1, 2500, 77, 128, 64, "f32"),
    gc.case("bf16_mixture", "mixture16", 4, 784, 784, 64, 64, "bf16"),
    gc.case("bf16_normclip", "normclip", 2, 2048, 200, 64, 96, "bf16"),
    gc.case("bf16_walk_d128", "walk", 2, 4100, 64, 128, 200, "bf16"),
    gc.case("bf16_iid_d128", "iid", 1, 5000, 300, 128, 128, "bf16"),
    gc.case("bf16_many_small", "iid", 300, 96, 40, 64, 8, "bf16"),
    gc.case("bf16_rank_chunks", "mixture16", 2, 1600, 1600, 64, 300, "bf16"),
]


@pytest.fixture(scope="module", autouse=True)
def _auto_cluster():
    wc.set_select_cluster(0)
    yield
    wc.set_select_cluster(0)


def test_pivot_uniforms_bit_exact(orc):
    """The device Philox draws are the oracle's, bit for bit, on 10^6 counters."""
    for seed in (0, 11, 2**63 + 12345):
        u_gpu = wc.pivot_uniforms(seed, 1000, 1000).cpu().numpy()
        u_orc = orc.pivot_uniforms(seed, 1000, 1000)
        assert np.array_equal(u_gpu, u_orc)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_stagewise_parity(orc, w):
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    # -- select (sampling) vs the oracle's own draws --
    S, F, rank, K_S = wc.select(d["K"], w.beta, w.r, w.pivot_seed, EPS)
    torch.cuda.synchronize()
    S_g, F_g, rank_g = S.cpu().numpy(), F.cpu().numpy(), rank.cpu().numpy()
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    compared = gc.pivots_agree_until_tie(S_g, own["S"], own["margin"], rank_g, own["rank"],
                                         F_g, own["F"], EPS)
    if w.dtype == "f32":
        assert all(c == rr for c, rr in zip(compared, rank_g)) or \
            np.nanmin(own["margin"]) < gc.TIE_MARGIN
    # structural facts of the device factor
    for b in range(w.BH):
        rr = rank_g[b]
        assert len(set(S_g[b, :rr].tolist())) == rr and np.all(S_g[b, rr:] == -1)
        assert np.all(F_g[b, rr:] == 0)
    # -- factor on the same pivots (the oracle follows the device's stopping step) --
    fx = orc.rpcholesky(ex["K"], w.beta, w.r, eps=0.0, S_fixed=S_g)
    assert np.array_equal(fx["rank"], rank_g)
    assert gc.column_rel_err(F_g, fx["F"], rank_g) < (2e-4 if w.dtype == "f32" else 2e-4)
    KS_ref = orc.gather(ex["K"], S_g, rank_g)
    assert np.array_equal(K_S.float().cpu().numpy().astype(np.float64), KS_ref)
    # -- weights --
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, d["V"])
    VS_o, w_o = orc.weights(fx["F"], S_g, rank_g, ex["V"])
    lo, hi = orc.value_range(ex["V"])
    assert np.array_equal(vmin.cpu().numpy(), lo) and np.array_equal(vmax.cpu().numpy(), hi)
    # -- attend, and the whole path against the oracle on the same pivots --
    O = wc.attend(d["Q"], K_S, rank, w.beta, V_S, wv, vmin, vmax).cpu().numpy()
    O_o, _, _ = orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, w.r, eps=0.0, S_fixed=S_g)
    assert np.all(O >= lo[:, None, :]) and np.all(O <= hi[:, None, :])
    assert gc.r12(O, O_o, lo, hi) <= gc.TOL_R12[w.dtype]
    assert wc.device_status() == 0
    # -- fused forward equals the staged calls bit for bit --
    O_f, S_f, rank_f = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, w.pivot_seed, EPS)
    assert torch.equal(S_f, S) and torch.equal(rank_f, rank)
    assert np.array_equal(O_f.cpu().numpy(), O)


# the triangular solve's shared-memory forms: the whole pivot block (r <= ~220),
# streamed in sub-blocks of 32 pivots (r <= 640; 4-byte copies when r % 4 != 0)
# and of 16 pivots (640 < r <= 1024)
SOLVE_CASES = [
    gc.case("solve_stream32_r250", "iid", 2, 1200, 16, 64, 250, "f32"),
    gc.case("solve_stream32_bf16_r512", "iid", 1, 2048, 16, 128, 512, "bf16"),
    gc.case("solve_stream16_r700", "walk", 1, 1500, 16, 64, 700, "bf16"),
    gc.case("solve_stream16_r900_truncated", "walk", 1, 8000, 16, 128, 900, "bf16"),  # rank 466
]


@pytest.mark.parametrize("w", [CASES[0], CASES[4], CASES[5]] + SOLVE_CASES, ids=lambda w: w.name)
def test_weights_kernel_alone(orc, w):
    """wildcat_weights on the oracle's own factor (rounded to float32) against
    the oracle's weights on exactly that rounded factor.  Bounds, relative to
    the largest entry: 1e-5 for float32 values (fp32 split-K sums and back
    substitution; measured <= 1.3e-6), 5e-5 for bfloat16 values (the factor
    split into bf16 hi + lo parts on the tensor cores, about 2^-17 relative
    per entry; measured <= 1.1e-5).  The SOLVE_CASES run the streamed forms
    of the back substitution (including a rank below r on the walk keys)."""
    dev, ex = workloads.make(w)
    res = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    F32 = res["F"].astype(np.float32)
    VS_o, w_o = orc.weights(F32.astype(np.float64), res["S"], res["rank"], ex["V"])
    V_S, wv, _, _ = wc.weights(torch.from_numpy(F32).cuda(), torch.from_numpy(res["S"]).cuda(),
                               torch.from_numpy(res["rank"]).cuda(), dev["V"].cuda())
    tol = 1e-5 if w.dtype == "f32" else 5e-5
    assert np.abs(V_S.cpu().numpy() - VS_o).max() <= tol * np.abs(VS_o).max()
    assert np.abs(wv.cpu().numpy() - w_o).max() <= tol * np.abs(w_o).max()


@pytest.mark.parametrize("w", [CASES[1], CASES[2], CASES[3], CASES[5], CASES[6]], ids=lambda w: w.name)
def test_attend_kernel_alone(orc, w):
    """wildcat_attend on the oracle's coreset (V_S, w rounded to float32)
    against the oracle's attend on the same rounded values.  float32 inputs
    run on CUDA cores in fp32; bfloat16 inputs with d in {64, 128} run on the
    tensor cores, where V_S and P are rounded to bfloat16 for the numerator's
    MMA and the denominator is summed in fp32 from the unrounded P."""
    dev, ex = workloads.make(w)
    res = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    VS_o, w_o = orc.weights(res["F"], res["S"], res["rank"], ex["V"])
    VS32, w32 = VS_o.astype(np.float32), w_o.astype(np.float32)
    lo, hi = orc.value_range(ex["V"])
    KS = orc.gather(ex["K"], res["S"], res["rank"])
    O_o = orc.attend(ex["Q"], KS, VS32.astype(np.float64), w32.astype(np.float64), res["rank"], lo,
                     hi, w.beta)
    KS_t = torch.from_numpy(KS).to(dev["K"].dtype).cuda()
    O = wc.attend(dev["Q"].cuda(), KS_t, torch.from_numpy(res["rank"]).cuda(), w.beta,
                  torch.from_numpy(VS32).cuda(), torch.from_numpy(w32).cuda(),
                  torch.from_numpy(lo.astype(np.float32)).cuda(),
                  torch.from_numpy(hi.astype(np.float32)).cuda()).cpu().numpy()
    assert wc.device_status() == 0
    assert gc.r12(O, O_o, lo, hi) <= gc.TOL_R12[w.dtype]


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_cluster_size_invariance(orc, G):
    """Any number of CTAs per instance gives the oracle's pivots (up to a
    near-tie) and the same factor."""
    w = gc.case("clusters", "iid", 3, 4096, 64, 64, 48, "f32")
    dev, ex = workloads.make(w)
    wc.set_select_cluster(G)
    try:
        S, F, rank, _ = wc.select(dev["K"].cuda(), w.beta, w.r, w.pivot_seed, EPS)
        torch.cuda.synchronize()
        assert wc.last_select_cluster() == G
    finally:
        wc.set_select_cluster(0)
    own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
    S_g, rank_g = S.cpu().numpy(), rank.cpu().numpy()
    gc.pivots_agree_until_tie(S_g, own["S"], own["margin"], rank_g, own["rank"],
                              F.cpu().numpy(), own["F"], EPS)
    fx = orc.rpcholesky(ex["K"], w.beta, w.r, eps=0.0, S_fixed=S_g)
    assert gc.column_rel_err(F.cpu().numpy(), fx["F"], rank_g) < 2e-4


def test_deterministic_across_calls():
    w = gc.case("det", "mixture16", 4, 784, 784, 64, 64, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    a = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 5)
    b = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 5)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 6)
    assert not torch.equal(a[1], c[1])


def test_duplicate_keys_truncate(orc):
    """Keys with only 5 distinct rows: the residual vanishes after 5 pivots,
    both sides stop at rank 5 and pad S, F, K_S, V_S, w."""
    rng = np.random.default_rng(3)
    base = rng.standard_normal((5, 64))
    K = base[rng.integers(0, 5, size=(2, 300))]
    Q = rng.standard_normal((2, 50, 64))
    V = rng.standard_normal((2, 300, 64))
    K32, Q32, V32 = (torch.from_numpy(x.astype(np.float32)) for x in (K, Q, V))
    S, F, rank, K_S = wc.select(K32.cuda(), 0.125, 12, 1, EPS)
    own = orc.rpcholesky(K32.double().numpy(), 0.125, 12, seed=1, eps=EPS)
    assert rank.cpu().tolist() == [5, 5] == own["rank"].tolist()
    assert np.all(S.cpu().numpy()[:, 5:] == -1)
    assert torch.all(F[:, 5:] == 0) and torch.all(K_S[:, 5:] == 0)
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, V32.cuda())
    assert torch.all(V_S[:, 5:] == 0) and torch.all(wv[:, 5:] == 0)
    O = wc.attend(Q32.cuda(), K_S, rank, 0.125, V_S, wv, vmin, vmax).cpu().numpy()
    O_o, _, _ = orc.wildcat_forward(Q32.double().numpy(), K32.double().numpy(),
                                    V32.double().numpy(), 0.125, 12, eps=EPS,
                                    S_fixed=S.cpu().numpy())
    lo, hi = orc.value_range(V32.double().numpy())
    assert gc.r12(O, O_o, lo, hi) <= 1e-4


def test_fixed_pivots_stop_and_rank_zero(orc):
    w = gc.case("fixed", "iid", 3, 200, 30, 32, 6, "f32")
    dev, ex = workloads.make(w)
    Sf = np.array([[5, 17, 3, 150, 9, 60], [1, 2, -1, 4, 5, 6], [-1] * 6], np.int32)
    S, F, rank, K_S = wc.select_fixed(dev["K"].cuda(), w.beta, torch.from_numpy(Sf).cuda(), EPS)
    assert rank.cpu().tolist() == [6, 2, 0]
    fx = orc.rpcholesky(ex["K"], w.beta, 6, eps=EPS, S_fixed=Sf)
    assert fx["rank"].tolist() == [6, 2, 0]
    assert gc.column_rel_err(F.cpu().numpy(), fx["F"], fx["rank"]) < 2e-4
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, dev["V"].cuda())
    O = wc.attend(dev["Q"].cuda(), K_S, rank, w.beta, V_S, wv, vmin, vmax).cpu().numpy()
    # rank 0: 0/0 is NaN, which the clip turns into v_min
    assert np.array_equal(O[2], np.broadcast_to(vmin.cpu().numpy()[2], O[2].shape))
    O_o, _, _ = orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, 6, eps=EPS, S_fixed=Sf)
    lo, hi = orc.value_range(ex["V"])
    assert gc.r12(O, O_o, lo, hi) <= 1e-4


def test_tensor_core_attend_rank_zero_and_short(orc):
    """bfloat16, d = 128 (the tensor-core attend): instances stopping after 6,
    2 and 0 fixed pivots, 300 queries (two query tiles, one partial).  Rank
    0 gives v_min everywhere; the others match the oracle on the same pivots."""
    w = gc.case("fixed_bf16", "iid", 3, 700, 300, 128, 6, "bf16")
    dev, ex = workloads.make(w)
    Sf = np.array([[5, 17, 3, 650, 9, 60], [1, 2, -1, 4, 5, 6], [-1] * 6], np.int32)
    S, F, rank, K_S = wc.select_fixed(dev["K"].cuda(), w.beta, torch.from_numpy(Sf).cuda(), EPS)
    assert rank.cpu().tolist() == [6, 2, 0]
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, dev["V"].cuda())
    O = wc.attend(dev["Q"].cuda(), K_S, rank, w.beta, V_S, wv, vmin, vmax).cpu().numpy()
    assert wc.device_status() == 0
    assert np.array_equal(O[2], np.broadcast_to(vmin.cpu().numpy()[2], O[2].shape))
    O_o, _, _ = orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, 6, eps=EPS, S_fixed=Sf)
    lo, hi = orc.value_range(ex["V"])
    assert gc.r12(O, O_o, lo, hi) <= gc.TOL_R12["bf16"]


def test_full_rank_recovers_exact_attention(orc):
    """r = n: the device estimate matches exact attention to float32 accuracy."""
    w = gc.case("full", "iid", 2, 48, 20, 32, 48, "f32", beta=0.25)
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 3, 1e-7)
    assert rank.cpu().tolist() == [48, 48]
    Oe = orc.exact_attention(ex["Q"], ex["K"], ex["V"], w.beta)
    lo, hi = orc.value_range(ex["V"])
    assert gc.r12(O.cpu().numpy(), Oe, lo, hi) <= 1e-4


def test_single_pivot_and_single_query(orc):
    """One pivot: P cancels in N / D, so the estimate is V_S / w for every
    query.  The tensor-core attend rounds V_S once to bfloat16 (relative
    error at most 2^-9, and |O| <= v_max - v_min here), which bounds the
    difference from the oracle."""
    w = gc.case("r1m1", "iid", 2, 130, 1, 64, 1, "bf16")
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward(d["Q"], d["K"], d["V"], w.beta, 1, 9)
    O_o, _, _ = orc.wildcat_forward(ex["Q"], ex["K"], ex["V"], w.beta, 1, eps=EPS,
                                    S_fixed=S.cpu().numpy())
    lo, hi = orc.value_range(ex["V"])
    assert gc.r12(O.cpu().numpy(), O_o, lo, hi) <= 2.0 ** -9


def test_forward_host_matches_device_forward():
    w = gc.case("host", "normclip", 2, 1500, 500, 64, 50, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O_d, S_d, r_d = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 4)
    pinned = {k: v.pin_memory() for k, v in dev.items()}
    O_h, S_h, r_h = wc.forward_host(pinned["Q"], pinned["K"], pinned["V"], w.beta, w.r, 4)
    assert torch.equal(O_h, O_d.cpu()) and torch.equal(S_h, S_d.cpu()) and torch.equal(r_h, r_d.cpu())


def test_shards_reproduce_the_whole_batch():
    """Instance sharding: each shard passes its first global instance as
    inst0, so two shards draw the pivots of the whole batch and give the
    same output bit for bit (run one after the other on one GPU)."""
    from nystr_coreset_approximate_b200 import sharding

    w = gc.case("shards", "iid", 7, 900, 100, 64, 24, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 7)
    parts = [sharding.forward_shard(d["Q"], d["K"], d["V"], w.beta, w.r, 7, 1e-6, 2, r)
             for r in range(2)]
    assert [p[3] for p in parts] == [0, 4]
    assert torch.equal(torch.cat([p[1] for p in parts]), S)
    assert torch.equal(torch.cat([p[2] for p in parts]), rank)
    assert torch.equal(torch.cat([p[0] for p in parts]), O)


def test_bounded_wait_reports_timeout_and_recovers():
    """A tensor-core wait that runs out (the test hook makes the attend wait
    on a barrier phase nothing completes, for 1 ms) is reported through the
    device status word; the context stays usable and the next call is clean."""
    w = gc.case("timeout", "mixture16", 2, 784, 784, 64, 64, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    S, F, rank, K_S = wc.select(d["K"], w.beta, w.r, 3)
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, d["V"])
    assert wc.device_status() == 0
    L = wc.lib()
    assert L.wildcat_test_force_wait_timeout(1_000_000) == 0
    try:
        wc.attend(d["Q"], K_S, rank, w.beta, V_S, wv, vmin, vmax)
        assert wc.device_status() == 5
    finally:
        assert L.wildcat_test_force_wait_timeout(0) == 0
    O = wc.attend(d["Q"], K_S, rank, w.beta, V_S, wv, vmin, vmax)
    assert wc.device_status() == 0
    assert torch.isfinite(O).all()


def test_concurrent_forwards_on_two_streams():
    """Two host threads run forwards at the same time, each on its own stream
    (the forwards fork their value range onto the library's per-device
    auxiliary stream under a per-device lock); every result equals the same
    forward run alone, bit for bit."""
    import threading

    cases = [gc.case("conc_plain", "iid", 4, 3000, 1000, 64, 64, "bf16"),
             gc.case("conc_binned", "normclip", 3, 4096, 700, 128, 96, "bf16", seed=9)]
    inputs, refs = [], []
    for k, w in enumerate(cases):
        dev, _ = workloads.make(w)
        d = gc.cuda_inputs(dev)
        inputs.append(d)
        if k == 0:
            refs.append(wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 5, EPS))
        else:
            refs.append(wc.forward_ex(d["Q"], d["K"], d["V"], w.beta, w.r, 5, EPS, nbins=2))
    torch.cuda.synchronize()
    out, errs = [None, None], []

    def run(k):
        try:
            w, d = cases[k], inputs[k]
            s = torch.cuda.Stream()
            res = []
            with torch.cuda.stream(s):
                for _ in range(6):
                    if k == 0:
                        r = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 5, EPS, stream=s)
                    else:
                        r = wc.forward_ex(d["Q"], d["K"], d["V"], w.beta, w.r, 5, EPS, nbins=2, stream=s)
                    res.append(r)
            s.synchronize()
            out[k] = res
        except Exception as e:  # reported below
            errs.append(e)

    th = [threading.Thread(target=run, args=(k,)) for k in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    assert wc.device_status() == 0
    for k in range(2):
        for O, S, rank in out[k]:
            assert torch.equal(S, refs[k][1]) and torch.equal(rank, refs[k][2]) and torch.equal(O, refs[k][0])


def test_forward_without_queries():
    """m = 0: the forward selects and forms the weights (pivots and ranks as
    with queries) and launches no attend; the host-buffer forward agrees."""
    w = gc.case("no_queries", "iid", 3, 1024, 64, 64, 48, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 3, EPS)
    Q0 = d["Q"][:, :0].contiguous()
    O0, S0, rank0 = wc.forward(Q0, d["K"], d["V"], w.beta, w.r, 3, EPS)
    assert O0.shape == (3, 0, 64)
    assert torch.equal(S0, S) and torch.equal(rank0, rank)
    Oe, Se, re_ = wc.forward_ex(Q0, d["K"], d["V"], w.beta, w.r, 3, EPS, nbins=2)
    assert Oe.shape == (3, 0, 64) and torch.all(re_ >= 1)
    assert wc.device_status() == 0
