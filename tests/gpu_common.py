"""Helpers shared by the GPU parity tests (device path vs the fp64 oracle)."""
from __future__ import annotations

import math

import numpy as np

import workloads

# Fixed-pivot parity bound on max_ij |O_gpu - O_oracle| / (v_max j - v_min j)
# (the benchmark spec's tolerance: 1e-4 for float32 inputs, 2e-2 for bfloat16).
TOL_R12 = {"f32": 1e-4, "bf16": 2e-2}
# A pivot draw whose u*T lands within this fraction of T from a bucket edge
# is a near-tie: fp32 (device) and fp64 (oracle) residuals may pick
# neighbouring buckets there, and every later pivot may differ.
TIE_MARGIN = 1e-4


def case(name, dist, BH, n, m, d, r, dtype, seed=7, pivot_seed=11, beta=None):
    return workloads.Workload(name=name, B=BH, H=1, n=n, m=m, d=d, r=r, dtype=dtype, dist=dist,
                              beta=beta if beta is not None else 1.0 / math.sqrt(d), seed=seed,
                              pivot_seed=pivot_seed)


def cuda_inputs(dev):
    return {k: v.cuda() for k, v in dev.items()}


def r12(O_a, O_b, vmin, vmax):
    """max over instances, rows, columns of |O_a - O_b| / (v_max j - v_min j)."""
    span = np.maximum(vmax - vmin, 1e-30)[:, None, :]
    return float(np.max(np.abs(np.asarray(O_a, np.float64) - O_b) / span))


def pivots_agree_until_tie(S_gpu, S_orc, margin, rank_gpu, rank_orc, F_gpu=None, F_orc=None,
                           eps=1e-6):
    """Pivot sequences must agree step by step until the oracle records a
    near-tie draw; returns the number of steps compared for each instance.

    With identical pivots the two sides may still stop at different steps
    when the pivot residual g_s sits at the truncation threshold eps (float32
    on the device, float64 in the oracle).  That is accepted only as a
    near-tie: the side that went on must have had g_s = F[i, s]^2 < 2 eps."""
    compared = []
    for b in range(S_gpu.shape[0]):
        k = 0
        upto = min(rank_gpu[b], rank_orc[b])
        while k < upto:
            if S_gpu[b, k] != S_orc[b, k]:
                assert margin[b, k] < TIE_MARGIN, (
                    f"instance {b}: pivots differ at step {k} ({S_gpu[b, k]} vs {S_orc[b, k]}) "
                    f"with oracle margin {margin[b, k]:.3e} (not a near-tie)")
                break
            k += 1
        if k == upto and rank_gpu[b] != rank_orc[b]:
            if rank_gpu[b] > rank_orc[b]:
                S, F = S_gpu, F_gpu
            else:
                S, F = S_orc, F_orc
            ok = False
            if F is not None:
                s = int(S[b, upto])
                gs = float(F[b, upto, s]) ** 2
                ok = gs < 2 * eps
            assert ok, (f"instance {b}: ranks differ ({rank_gpu[b]} vs {rank_orc[b]}) with "
                        "identical pivots and no truncation near-tie")
        compared.append(k)
    return compared


def column_rel_err(F_gpu, F_orc, rank):
    """max over factor columns i < rank of max_l |dF| / max_l |F_orc|."""
    worst = 0.0
    for b in range(F_gpu.shape[0]):
        for i in range(int(rank[b])):
            ref = F_orc[b, i]
            scale = max(np.abs(ref).max(), 1e-30)
            worst = max(worst, float(np.abs(F_gpu[b, i] - ref).max() / scale))
    return worst


def binned_pivots_agree_until_tie(orc, K, beta, r, nbins, seed, eps, S_gpu, rank_gpu, recenter=False, tau=1.0):
    """Free draws of the binned forward against the oracle's own draws, bin by
    bin, with the near-tie rule of pivots_agree_until_tie.  Bin q of instance b
    is the oracle's instance b * nbins + q of the [BH * nbins, n / nbins] view
    of the keys (recentred by the instance's mean over all n keys when asked),
    drawn with the key kernel exp(beta <x, y> / tau^2).  Returns the steps
    compared per bin."""
    BH, n, d = K.shape
    nb, rb = n // nbins, r // nbins
    Kx = K - K.mean(axis=1, keepdims=True) if recenter else K
    Kv = np.ascontiguousarray(Kx.reshape(BH * nbins, nb, d))
    beta_key = beta / (tau * tau)
    own = orc.rpcholesky(Kv, beta_key, rb, seed=seed, eps=eps)
    S_loc = np.asarray(S_gpu).reshape(BH, nbins, rb).copy()
    for q in range(nbins):
        valid = S_loc[:, q] >= 0
        S_loc[:, q][valid] -= q * nb
    S_loc = S_loc.reshape(BH * nbins, rb)
    rank_loc = np.asarray(rank_gpu).reshape(BH * nbins)
    # the factor on the device's pivots (for a stop at the truncation threshold)
    fx = orc.rpcholesky(Kv, beta_key, rb, eps=0.0, S_fixed=S_loc)
    return pivots_agree_until_tie(S_loc, own["S"], own["margin"], rank_loc, own["rank"], fx["F"], own["F"], eps)
