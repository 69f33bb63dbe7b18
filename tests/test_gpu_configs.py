"""The five workloads at full size, in the launch configuration the benchmark
times (one wildcat_forward over all instances through a preallocated
workspace), against the fp64 oracle.

- Fixed-pivot parity: on sampled instances (every instance of the ViT and
  image-generation workloads) and 256 sampled query rows, the
  oracle runs on the device's pivots (and stops where the device stopped);
  max |O_gpu - O_oracle| / (v_max - v_min) <= 1e-4 (float32) / 2e-2 (bfloat16).
- Error against exact attention (oracle, float64) on the same rows: the
  device's error is within 1.1x of the oracle's (plus 1e-6 of the value
  range for float32 rounding).
- Pivots: bit-exact on the float32 unit workload; elsewhere equal to the
  oracle's own draws until a near-tie where the oracle's draw is affordable.
"""
import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

EPS = 1e-6

# instances checked against the oracle, and whether the oracle also draws its
# own pivots for the whole batch (cheap enough below ~10 s)
PLAN = {
    "c0_unit": ([0], True),
    "c1_vit56": (list(range(32)), True),
    "c2_imggen64": (list(range(128)), True),
    "c3_kvcache": ([0, 31], False),
    "c4a_long16k": ([0, 7], False),
    "c4b_long64k": ([0, 7], False),
    "c4c_long128k": ([0, 7], False),
}


@pytest.mark.parametrize("name", list(PLAN), ids=list(PLAN))
def test_full_size_config(orc, name):
    w = workloads.CONFIGS[name]
    insts, own_draws = PLAN[name]
    dev, ex = workloads.make(w)
    Q, K, V = (dev[k].cuda() for k in ("Q", "K", "V"))
    plan = wc.ForwardPlan(w.BH, w.m, w.n, w.d, w.r, w.dtype)
    O, S, rank = plan.run(Q, K, V, w.beta, w.pivot_seed, EPS)
    torch.cuda.synchronize()
    O, S, rank = O.cpu().numpy(), S.cpu().numpy(), rank.cpu().numpy()
    del Q, K, V, plan
    torch.cuda.empty_cache()
    assert np.all(rank >= 1)
    for b in range(w.BH):
        rr = rank[b]
        assert len(set(S[b, :rr].tolist())) == rr and np.all(S[b, rr:] == -1)

    rows = np.arange(w.m) if name == "c0_unit" else workloads.sample_rows(w, 256)
    sub = {k: ex[k][insts] for k in ("Q", "K", "V")}
    O_fix, _, rank_fix = orc.wildcat_forward(sub["Q"], sub["K"], sub["V"], w.beta, w.r, eps=0.0,
                                             S_fixed=S[insts], rows=rows)
    assert np.array_equal(rank_fix, rank[insts])
    lo, hi = orc.value_range(sub["V"])
    O_gpu = O[insts][:, rows]
    assert np.all(O_gpu >= lo[:, None, :]) and np.all(O_gpu <= hi[:, None, :])
    metric = gc.r12(O_gpu, O_fix, lo, hi)
    assert metric <= gc.TOL_R12[w.dtype], metric

    O_ex = orc.exact_attention(sub["Q"], sub["K"], sub["V"], w.beta, rows=rows)
    err_gpu = float(np.abs(O_gpu - O_ex).max())
    err_orc = float(np.abs(O_fix - O_ex).max())
    slack = 1e-6 * float((hi - lo).max())
    assert err_gpu <= 1.1 * err_orc + slack, (err_gpu, err_orc)

    if own_draws:
        own = orc.rpcholesky(ex["K"], w.beta, w.r, seed=w.pivot_seed, eps=EPS)
        if name == "c0_unit":
            # float32 unit workload: pivot indices bit-exact
            assert np.array_equal(S, own["S"]) and np.array_equal(rank, own["rank"]), \
                f"min draw margin {np.nanmin(own['margin']):.3e}"
        else:
            gc.pivots_agree_until_tie(S, own["S"], own["margin"], rank, own["rank"], None,
                                      own["F"], EPS)
