"""The inverse-maintenance weights route (wildcat_weights_inverse) against the
fp64 oracle's inverse route on the device's own pivots.

Both sides run in fp64 from the same inputs (bfloat16 / float32 values
widened exactly) and differ only in summation order, so the bound is tight:
max |(V_S, w)_gpu - (V_S, w)_oracle| <= 1e-6 * max |(V_S, w)_oracle| per
instance (fp64 rounding amplified by the condition number of h(K_S, K_S),
at most 1 / eps = 1e6 after truncation, then one rounding to float32).
The value range is bit-exact.  The factor route (float32 on the device)
must agree with the inverse route where h(K_S, K_S) is well conditioned.
The cases cover the inverse held by one CTA (r up to about 160), spread over
clusters of 2, 4 and 16 CTAs (ragged row blocks and truncation included),
and held in global memory (r = 700).
"""
import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

EPS = 1e-6

CASES = [
    gc.case("inv_f32_d64", "iid", 3, 1000, 16, 64, 40, "f32"),
    gc.case("inv_bf16_mix", "mixture16", 2, 1568, 1568, 64, 96, "bf16"),
    gc.case("inv_bf16_d128", "iid", 2, 3000, 16, 128, 130, "bf16"),
    gc.case("inv_f32_d32_ragged", "iid", 2, 777, 16, 32, 33, "f32"),
    gc.case("inv_walk_trunc", "walk", 2, 4096, 16, 128, 300, "bf16"),        # clusters of 4, truncated
    gc.case("inv_cluster2", "iid", 2, 2048, 16, 64, 200, "bf16"),            # clusters of 2
    gc.case("inv_cluster4_ragged", "iid", 3, 2500, 16, 64, 250, "f32"),      # 63 rows per CTA, last 61
    gc.case("inv_cluster16", "iid", 2, 4096, 16, 128, 512, "bf16"),          # clusters of 16
    gc.case("inv_global", "iid", 1, 2048, 16, 64, 700, "bf16"),              # inverse in global memory
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_inverse_route_matches_oracle(orc, w):
    dev, ex = workloads.make(w)
    K, V = dev["K"].cuda(), dev["V"].cuda()
    S, F, rank, _ = wc.select(K, w.beta, w.r, w.pivot_seed, EPS)
    V_S, wv, vmin, vmax = wc.weights_inverse(K, S, rank, V, w.beta)
    torch.cuda.synchronize()
    S_h, rank_h = S.cpu().numpy(), rank.cpu().numpy()
    VS_o, w_o = orc.weights_inverse(ex["K"], S_h, rank_h, ex["V"], w.beta)
    got = np.concatenate([V_S.cpu().numpy(), wv.cpu().numpy()[:, :, None]], axis=2)
    ref = np.concatenate([VS_o, w_o[:, :, None]], axis=2)
    for b in range(w.BH):
        scale = np.abs(ref[b]).max()
        assert np.abs(got[b] - ref[b]).max() <= 1e-6 * scale
        assert np.all(got[b, rank_h[b]:] == 0)
    lo, hi = orc.value_range(ex["V"])
    assert np.array_equal(vmin.cpu().numpy(), lo) and np.array_equal(vmax.cpu().numpy(), hi)
    assert wc.device_status() == 0


def test_inverse_route_equals_factor_route_when_well_conditioned(orc):
    """Few well-separated pivots: both device routes give the same weights
    (the factor route in float32) and the same attention output."""
    w = gc.case("inv_vs_factor", "iid", 2, 2048, 128, 64, 24, "f32")
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    S, F, rank, K_S = wc.select(d["K"], w.beta, w.r, w.pivot_seed, EPS)
    VS_f, w_f, lo, hi = wc.weights(F, S, rank, d["V"])
    VS_i, w_i, lo_i, hi_i = wc.weights_inverse(d["K"], S, rank, d["V"], w.beta)
    assert torch.equal(lo, lo_i) and torch.equal(hi, hi_i)
    scale = VS_i.abs().max().item()
    assert (VS_f - VS_i).abs().max().item() <= 1e-3 * scale
    O_f = wc.attend(d["Q"], K_S, rank, w.beta, VS_f, w_f, lo, hi)
    O_i = wc.attend(d["Q"], K_S, rank, w.beta, VS_i, w_i, lo, hi)
    span = (hi - lo).max().item()
    assert (O_f - O_i).abs().max().item() <= 1e-3 * span


def test_inverse_route_rank_zero_and_one(orc):
    """rank 0 gives zero weights; rank 1 is the closed form
    W = h(k_s, K) / h(k_s, k_s)."""
    w = gc.case("inv_r1", "iid", 2, 512, 16, 32, 4, "f32")
    dev, ex = workloads.make(w)
    K, V = dev["K"].cuda(), dev["V"].cuda()
    S = torch.tensor([[5, -1, -1, -1], [300, -1, -1, -1]], dtype=torch.int32, device="cuda")
    rank = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    V_S, wv, _, _ = wc.weights_inverse(K, S, rank, V, w.beta)
    V_S, wv = V_S.cpu().numpy(), wv.cpu().numpy()
    assert np.all(V_S[1] == 0) and np.all(wv[1] == 0) and np.all(V_S[0, 1:] == 0)
    Kx, Vx = ex["K"][0], ex["V"][0]
    h = np.exp(w.beta * (Kx @ Kx[5]))
    hss = np.exp(w.beta * (Kx[5] @ Kx[5]))
    np.testing.assert_allclose(V_S[0, 0], h @ Vx / hss, rtol=1e-6, atol=1e-6 * np.abs(h @ Vx / hss).max())
    np.testing.assert_allclose(wv[0, 0], h.sum() / hss, rtol=1e-6)
