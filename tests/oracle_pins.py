"""Pins for the fp64 oracle: checks against facts fixed by the method's
definitions and by mathematics, never against the oracle itself.

Source of every definition: "WildCat: Near-Linear Attention in Theory and
Practice", Sec. 2 (exponential kernel h, plug-in estimator with value-range
clip, Nystrom weights W = h(K_S,K_S)^+ h(K_S,K), randomly pivoted Cholesky
sampling from the residual diagonal, rank-one inverse update of
h(K_S,K_S)^-1, invariance under key recentring).

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
on failure.  ``tests/test_oracle_pins.py`` runs them on the real oracle;
``tests/test_oracle_mutants.py`` runs them on copies of the oracle with one
planted mistake each and requires every copy to fail at least one pin.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
from scipy import special, stats

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(seed, BH, m, n, d, scale=1.0):
    rng = np.random.default_rng(seed)
    return (scale * rng.standard_normal((BH, m, d)), scale * rng.standard_normal((BH, n, d)),
            rng.standard_normal((BH, n, d)))


def _H(K, beta):
    """Key kernel matrix h(K, K) = exp(beta K K^T), one instance, by numpy."""
    return np.exp(beta * K @ K.T)


def _W_of(o, F, S, rank, n):
    """The n-column weight matrix W itself: W I_n through the oracle's weights."""
    BH = F.shape[0]
    eye = np.broadcast_to(np.eye(n), (BH, n, n)).copy()
    W, w = o.weights(F, S, rank, eye)
    return W, w


# --------------------------------------------------------------------------- P1
def pin_exact_bruteforce(o):
    """P1: exact attention equals softmax(beta Q K^T) V by scipy, rows of the
    softmax matrix sum to one, outputs lie in the value range."""
    Q, K, V = _rand(11, 3, 7, 13, 5, scale=1.5)
    beta = 0.7
    O = o.exact_attention(Q, K, V, beta)
    for b in range(3):
        P = special.softmax(beta * Q[b] @ K[b].T, axis=1)
        np.testing.assert_allclose(P.sum(1), 1.0, rtol=0, atol=1e-14)
        np.testing.assert_allclose(O[b], P @ V[b], rtol=0, atol=1e-13)
        assert np.all(O[b] >= V[b].min(0) - 1e-14) and np.all(O[b] <= V[b].max(0) + 1e-14)
    rows = np.array([6, 0, 3])
    np.testing.assert_allclose(o.exact_attention(Q, K, V, beta, rows=rows), O[:, rows], 0, 0)


# --------------------------------------------------------------------------- P2
def pin_full_rank_is_exact(o):
    """P2: with r = n every key is a pivot, W is a permutation, and the
    plug-in estimate equals exact attention to 1e-9."""
    for (n, d, beta, seed) in [(16, 8, 0.5, 1), (32, 8, 0.25, 2), (12, 4, 0.5, 3)]:
        Q, K, V = _rand(100 + seed, 2, 9, n, d)
        O, S, rank = o.wildcat_forward(Q, K, V, beta, n, seed=seed, eps=1e-14)
        assert np.all(rank == n), rank
        assert all(sorted(S[b].tolist()) == list(range(n)) for b in range(2))
        np.testing.assert_allclose(O, o.exact_attention(Q, K, V, beta), rtol=0, atol=1e-9)


# --------------------------------------------------------------------------- P3
def pin_weights_textbook_solve(o):
    """P3: for fixed pivots, the factor route W (V,1) equals
    h(K_S,K_S)^-1 h(K_S,K) (V,1) from a dense LU solve (numpy.linalg.solve)."""
    n, d, r, beta = 40, 6, 9, 0.4
    _, K, V = _rand(21, 2, 1, n, d)
    S_fixed = np.array([[3, 17, 5, 39, 0, 22, 11, 30, 8], [1, 2, 3, 4, 5, 6, 7, 8, 9]], np.int32)
    res = o.rpcholesky(K, beta, r, eps=1e-14, S_fixed=S_fixed)
    assert np.all(res["rank"] == r)
    np.testing.assert_array_equal(res["S"], S_fixed)
    VS, w = o.weights(res["F"], res["S"], res["rank"], V)
    for b in range(2):
        H = _H(K[b], beta)
        s = S_fixed[b]
        Wt = np.linalg.solve(H[np.ix_(s, s)], H[s, :])
        ref = Wt @ np.concatenate([V[b], np.ones((n, 1))], axis=1)
        got = np.concatenate([VS[b], w[b][:, None]], axis=1)
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10 * np.abs(ref).max())


# --------------------------------------------------------------------------- P4
def _rpnys_inverse_route(K, beta, r, uniform, eps):
    """RPNys with the rank-one inverse update (Sec. 2: g = (h(k_s,K_S)
    h(K_S,K_S)^-1, -1) / sqrt(h_res(k_s,k_s)), inverse <- [[inv,0],[0,0]] + g g^T),
    written independently of the oracle.  Returns (S, W, diag history)."""
    n = K.shape[0]
    H = _H(K, beta)
    diag = np.diag(H).copy()
    S, hist = [], []
    inv = np.zeros((0, 0))
    for i in range(r):
        diag = np.maximum(diag, 0.0)
        hist.append(diag.copy())
        T = diag.sum()
        if not T > 0:
            break
        t = uniform(i) * T
        s = int(np.searchsorted(np.cumsum(diag), t, side="left"))
        hs = H[s, S] if S else np.zeros(0)
        res_col = H[:, s] - (H[:, S] @ (inv @ hs) if S else 0.0)  # h_res(k_l, k_s)
        res_ss = res_col[s]
        if not res_ss > eps * np.diag(H).max():
            break
        g = np.concatenate([hs @ inv if S else np.zeros(0), [-1.0]]) / math.sqrt(res_ss)
        grown = np.zeros((len(S) + 1, len(S) + 1))
        grown[:len(S), :len(S)] = inv
        inv = grown + np.outer(g, g)
        diag = diag - res_col ** 2 / res_ss
        diag[s] = 0.0
        S.append(s)
    W = inv @ H[S, :]
    return S, W, hist


def pin_inverse_update_route(o):
    """P4: pivots, weights and residual diagonals agree with the rank-one
    inverse-update derivation of RPNys drawing the same uniforms."""
    n, d, r, beta, seed = 48, 5, 10, 0.3, 77
    _, K, V = _rand(31, 2, 1, n, d)
    res = o.rpcholesky(K, beta, r, seed=seed, eps=1e-13, shift=False, history=True)
    W, _ = _W_of(o, res["F"], res["S"], res["rank"], n)
    for b in range(2):
        S, Wi, hist = _rpnys_inverse_route(K[b], beta, r, lambda i: o.pivot_uniform(seed, i, b),
                                           1e-13)
        assert res["rank"][b] == len(S)
        np.testing.assert_array_equal(res["S"][b][:len(S)], S)
        np.testing.assert_allclose(W[b][:len(S)], Wi, rtol=0, atol=1e-9 * np.abs(Wi).max())
        for i, h in enumerate(hist):
            np.testing.assert_allclose(res["hist"][b][i], h, rtol=1e-9, atol=1e-12 * h.max())


# --------------------------------------------------------------------------- P5
def pin_partial_cholesky_interpolates(o):
    """P5: F F^T reproduces the (shifted) kernel on the pivot columns, W is the
    identity on the pivots, the residual diagonal is diag(H) - |F_l|^2 and
    vanishes on the pivots."""
    n, d, r, beta, seed = 60, 7, 12, 0.35, 5
    _, K, _ = _rand(41, 2, 1, n, d)
    res = o.rpcholesky(K, beta, r, seed=seed, eps=1e-13, history=True)
    W, w = _W_of(o, res["F"], res["S"], res["rank"], n)
    for b in range(2):
        rr = res["rank"][b]
        assert rr == r
        S = res["S"][b][:rr]
        sq = (K[b] ** 2).sum(1)
        Hs = np.exp(beta * (K[b] @ K[b].T - sq.max()))
        F = res["F"][b][:rr].T  # n x r
        np.testing.assert_allclose((F @ F.T)[:, S], Hs[:, S], rtol=0, atol=1e-12)
        np.testing.assert_allclose(W[b][:rr][:, S], np.eye(rr), rtol=0, atol=1e-10)
        for i in range(rr + 1):
            expect = np.maximum(np.diag(Hs) - (F[:, :i] ** 2).sum(1), 0.0)
            expect[S[:i]] = 0.0
            np.testing.assert_allclose(res["hist"][b][i], expect, rtol=0, atol=1e-12)
        # lower-triangular pivot block: F_{S_a, j} = 0 for j > a (up to rounding)
        FS = F[S, :]
        assert np.abs(np.triu(FS, 1)).max() < 1e-12


# --------------------------------------------------------------------------- P6
def pin_residual_invariants(o):
    """P6: residual diagonal non-negative and non-increasing, its trace strictly
    decreasing, pivots distinct (iid and clustered keys)."""
    for seed, clustered in [(1, False), (2, True)]:
        rng = np.random.default_rng(50 + seed)
        n, d, r, beta = 200, 8, 40, 0.5
        if clustered:
            c = rng.standard_normal((4, d))
            K = c[rng.integers(0, 4, n)] + 0.3 * rng.standard_normal((n, d))
        else:
            K = rng.standard_normal((n, d))
        res = o.rpcholesky(K[None], beta, r, seed=seed, eps=1e-12, history=True)
        rr = res["rank"][0]
        h = res["hist"][0][:rr + 1]
        assert np.all(h >= 0)
        assert np.all(np.diff(h, axis=0) <= 1e-12 * h[0].max())
        tr = h.sum(1)
        assert np.all(np.diff(tr) < 0)
        S = res["S"][0][:rr]
        assert len(set(S.tolist())) == rr and np.all(res["S"][0][rr:] == -1)
        for i, s in enumerate(S):
            assert h[i][s] > 0, "a zero-mass index was drawn"


# --------------------------------------------------------------------------- P7
def _triton_philox(ctrs, keys):
    """Philox4x32-10 from the triton library, run by its CPU interpreter."""
    os.environ["TRITON_INTERPRET"] = "1"
    import torch
    import triton
    import triton.language as tl

    @triton.jit
    def _k(c0p, c1p, c2p, c3p, out, seed, N: tl.constexpr):
        i = tl.arange(0, N)
        a, b, c, d = tl.philox(seed, tl.load(c0p + i), tl.load(c1p + i), tl.load(c2p + i),
                               tl.load(c3p + i))
        tl.store(out + i * 4, a)
        tl.store(out + i * 4 + 1, b)
        tl.store(out + i * 4 + 2, c)
        tl.store(out + i * 4 + 3, d)

    outs = []
    for ctr, key in zip(ctrs, keys):
        cols = [torch.tensor([c], dtype=torch.int64).to(torch.uint32) for c in ctr]
        out = torch.zeros(4, dtype=torch.int64).to(torch.uint32)
        seed = (int(key[1]) << 32) | int(key[0])
        _k[(1,)](*cols, out, seed, N=1)
        outs.append([int(x) & 0xFFFFFFFF for x in out.to(torch.int64).tolist()])
    return outs


def pin_philox_matches_library(o):
    """P7a: the oracle's Philox4x32-10 equals the triton library's Philox
    (CPU interpreter) on assorted counters and keys, incl. all-ones words."""
    ctrs = [(0, 0, 0, 0), (1, 0, 0, 0), (5, 3, 0, 0), (0xFFFFFFFF,) * 4,
            (0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (127, 31, 0, 0)]
    keys = [(0, 0), (0, 0), (7, 0), (0xFFFFFFFF, 0xFFFFFFFF), (0xA4093822, 0x299F31D0),
            (0x89ABCDEF, 0x01234567)]
    want = _triton_philox(ctrs, keys)
    got = [o.philox4x32_10(c, k) for c, k in zip(ctrs, keys)]
    assert got == want, (got, want)


def pin_uniform_mapping_matches_library(o):
    """P7a': the pivot uniform of (seed, step, instance) is the triton
    library's Philox4x32-10 run with that 64-bit seed (the library splits it
    into the key words itself) on counter (step, instance, 0, 0), its first
    two words joined high:low and cut to 53 bits, plus one, times 2^-53."""
    cases = [(0x0123456789ABCDEF, 0, 0), (0x0123456789ABCDEF, 5, 3), (7, 127, 31),
             (0xFEDCBA9876543210, 1, 2**31 - 1)]
    ctrs = [(step, inst, 0, 0) for _, step, inst in cases]
    keys = [(seed & 0xFFFFFFFF, seed >> 32) for seed, _, _ in cases]
    for (seed, step, inst), x in zip(cases, _triton_philox(ctrs, keys)):
        bits = ((x[1] << 32) | x[0]) >> 11
        assert o.pivot_uniform(seed, step, inst) == (bits + 1) * 2.0 ** -53, (seed, step, inst)


def pin_uniforms_uniform(o):
    """P7b: the pivot uniforms lie in (0, 1] and pass a Kolmogorov-Smirnov test."""
    u = np.array([o.pivot_uniform(9, i, b) for i in range(400) for b in range(50)])
    assert np.all(u > 0) and np.all(u <= 1)
    assert stats.kstest(u, "uniform").pvalue > 1e-3


def pin_first_pivot_law(o):
    """P7c: over many seeds the first pivot is distributed proportionally to
    the initial diagonal h(k_l, k_l) (chi-square test)."""
    rng = np.random.default_rng(61)
    n, d, beta = 8, 3, 0.6
    K = rng.standard_normal((1, n, d)) * np.linspace(0.3, 1.6, n)[None, :, None]
    p = np.exp(beta * (K[0] ** 2).sum(1))
    p /= p.sum()
    counts = np.zeros(n)
    for seed in range(6000):
        counts[o.rpcholesky(K, beta, 1, seed=seed, eps=1e-12)["S"][0, 0]] += 1
    assert stats.chisquare(counts, p * counts.sum()).pvalue > 1e-4


# --------------------------------------------------------------------------- P8
def pin_shift_invariance(o):
    """P8: the global shift M_K changes neither pivots nor weights."""
    n, d, r, beta = 50, 6, 12, 0.45
    _, K, V = _rand(71, 2, 1, n, d, scale=1.3)
    a = o.rpcholesky(K, beta, r, seed=4, eps=1e-13, shift=True)
    b = o.rpcholesky(K, beta, r, seed=4, eps=1e-13, shift=False)
    np.testing.assert_array_equal(a["S"], b["S"])
    Wa, wa = o.weights(a["F"], a["S"], a["rank"], V)
    Wb, wb = o.weights(b["F"], b["S"], b["rank"], V)
    np.testing.assert_allclose(Wa, Wb, rtol=0, atol=1e-12 * np.abs(Wb).max())
    np.testing.assert_allclose(wa, wb, rtol=0, atol=1e-12 * np.abs(wb).max())


# --------------------------------------------------------------------------- P9
def pin_value_range_and_recentring(o):
    """P9: every plug-in output lies in [v_min j, v_max j] (also when the
    estimated normaliser goes negative); recentring the keys leaves exact
    attention unchanged."""
    Q, K, V = _rand(81, 3, 40, 120, 6, scale=1.2)
    beta = 0.8
    O, S, rank = o.wildcat_forward(Q, K, V, beta, 6, seed=2)
    vmin, vmax = o.value_range(V)
    assert np.all(O >= vmin[:, None, :]) and np.all(O <= vmax[:, None, :])
    np.testing.assert_array_equal(vmin, V.min(1))
    np.testing.assert_array_equal(vmax, V.max(1))
    Kc = K - K.mean(axis=1, keepdims=True)
    np.testing.assert_allclose(o.exact_attention(Q, Kc, V, beta), o.exact_attention(Q, K, V, beta),
                               rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- P10
def pin_error_falls_with_rank(o):
    """P10: median error against exact attention falls as the coreset grows."""
    errs = []
    for r in (4, 16, 48):
        e = []
        for seed in range(5):
            Q, K, V = _rand(90 + seed, 1, 64, 256, 8)
            O, _, _ = o.wildcat_forward(Q, K, V, 0.35, r, seed=seed)
            e.append(np.abs(O - o.exact_attention(Q, K, V, 0.35)).max())
        errs.append(np.median(e))
    assert errs[0] > errs[1] > errs[2], errs


# --------------------------------------------------------------------------- closed forms
def pin_single_pivot_closed_form(o):
    """With one fixed pivot s, W = h(k_s,k_s)^-1 h(k_s,K), so the estimate
    is the query-independent kernel-weighted mean
    sum_l e^{beta<k_s,k_l>} v_l / sum_l e^{beta<k_s,k_l>}, clipped."""
    Q, K, V = _rand(95, 2, 11, 30, 4)
    beta = 0.6
    S_fixed = np.array([[7], [0]], np.int32)
    O, S, rank = o.wildcat_forward(Q, K, V, beta, 1, S_fixed=S_fixed)
    for b in range(2):
        a = np.exp(beta * K[b] @ K[b][S_fixed[b, 0]])
        mean = (a @ V[b]) / a.sum()
        expect = np.clip(mean, V[b].min(0), V[b].max(0))
        np.testing.assert_allclose(O[b], np.broadcast_to(expect, O[b].shape), rtol=0, atol=1e-13)


def pin_hand_examples(o):
    """Hand-worked examples stored in tests/golden/hand_examples.json."""
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        Q = np.array(c["Q"], float)[None]
        K = np.array(c["K"], float)[None]
        V = np.array(c["V"], float)[None]
        beta = float(eval(c["beta"], {"math": math}))
        Sf = np.array([c["S"]], np.int32)
        O, _, rank = o.wildcat_forward(Q, K, V, beta, len(c["S"]), S_fixed=Sf, eps=1e-14)
        np.testing.assert_allclose(O[0], np.array(c["O_hat"], float), rtol=0, atol=1e-12,
                                   err_msg=c["name"])
        if "O_exact" in c:
            np.testing.assert_allclose(o.exact_attention(Q, K, V, beta)[0],
                                       np.array(c["O_exact"], float), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- binning
def pin_binning_closed_forms(o):
    """Divide-and-conquer binning (Sec. 2): one bin is the unbinned method
    bit for bit; r = n (every key a pivot of its bin) makes every bin's
    weights a permutation, so the union estimate is exact attention; pivots
    of bin q lie inside bin q and are distinct."""
    Q, K, V = _rand(131, 2, 20, 48, 6)
    a = o.wildcat_forward(Q, K, V, 0.4, 12, seed=3)
    b1 = o.wildcat_forward_binned(Q, K, V, 0.4, 12, 1, seed=3)
    np.testing.assert_array_equal(a[0], b1[0])
    np.testing.assert_array_equal(a[1], b1[1])
    O, S, rank = o.wildcat_forward_binned(Q, K, V, 0.4, 48, 4, seed=3, eps=1e-14)
    assert np.all(rank == 12)
    np.testing.assert_allclose(O, o.exact_attention(Q, K, V, 0.4), rtol=0, atol=1e-12)
    O, S, rank = o.wildcat_forward_binned(Q, K, V, 0.4, 16, 4, seed=5)
    for b in range(2):
        for q in range(4):
            rows = S[b, 4 * q:4 * q + rank[b, q]]
            assert np.all((rows >= 12 * q) & (rows < 12 * q + 12))
        valid = S[b][S[b] >= 0]
        assert len(set(valid.tolist())) == len(valid)


def pin_binning_composes_unbinned_parts(o):
    """Binning as a second derivation from the unbinned primitives (Sec. 2,
    divide and conquer): select and weights on the [BH * nbins, n / nbins]
    view of K and V (bin q of instance b is instance b * nbins + q, which is
    also its Philox counter word), the union coreset puts the bins' pivot
    rows and weights side by side (zero rows past a bin's rank), and the
    attend over it clips to the value range of all n values.  The binned
    forward gives the same pivots, ranks and output.  Bin q's values are
    offset by 3 q, so the union's estimates mix bins and lie outside any one
    bin's range (a clip to one bin's range would show)."""
    Q, K, V = _rand(161, 2, 20, 48, 6)
    beta, r, nb, seed = 0.4, 16, 4, 7
    BH, n, d = K.shape
    rb, nbk = r // nb, n // nb
    V = V + 3.0 * (np.arange(n) // nbk)[None, :, None]
    O, S, rank = o.wildcat_forward_binned(Q, K, V, beta, r, nb, seed=seed)
    Kv, Vv = K.reshape(BH * nb, nbk, d), V.reshape(BH * nb, nbk, d)
    res = o.rpcholesky(Kv, beta, rb, seed=seed)
    np.testing.assert_array_equal(rank.reshape(-1), res["rank"])
    for b in range(BH):
        for q in range(nb):
            rr = res["rank"][b * nb + q]
            np.testing.assert_array_equal(S[b, q * rb:q * rb + rr], q * nbk + res["S"][b * nb + q, :rr])
            assert np.all(S[b, q * rb + rr:(q + 1) * rb] == -1)
    VS, w = o.weights(res["F"], res["S"], res["rank"], Vv)
    KS = o.gather(Kv, res["S"], res["rank"])
    lo, hi = o.value_range(V)
    O2 = o.attend(Q, KS.reshape(BH, r, d), VS.reshape(BH, r, d), w.reshape(BH, r),
                  np.full(BH, r, np.int32), lo, hi, beta)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- decode
def pin_decode_closed_form(o):
    """KV-cache decode: with the cache compressed at full rank (r = n, W a
    permutation), new token i attends exactly over all n cached keys and
    the new keys j <= i (causal softmax by numpy); with no cache rows
    (rank 0) it is plain causal attention among the new tokens."""
    rng = np.random.default_rng(141)
    BH, n, m, d, beta = 2, 24, 7, 5, 0.45
    K, V = rng.standard_normal((BH, n, d)), rng.standard_normal((BH, n, d))
    Qn, Kn, Vn = (rng.standard_normal((BH, m, d)) for _ in range(3))
    res = o.rpcholesky(K, beta, n, seed=2, eps=1e-14)
    assert np.all(res["rank"] == n)
    VS, w = o.weights(res["F"], res["S"], res["rank"], V)
    KS = o.gather(K, res["S"], res["rank"])
    lo, hi = o.value_range(V)
    O = o.decode_attend(Qn, Kn, Vn, KS, VS, w, res["rank"], lo, hi, beta)
    for b in range(BH):
        for i in range(m):
            keys = np.concatenate([K[b], Kn[b, :i + 1]])
            vals = np.concatenate([V[b], Vn[b, :i + 1]])
            p = special.softmax(beta * keys @ Qn[b, i])
            np.testing.assert_allclose(O[b, i], p @ vals, rtol=0, atol=1e-9)
    zero = np.zeros(BH, np.int32)
    O0 = o.decode_attend(Qn, Kn, Vn, KS, VS, w, zero, lo, hi, beta)
    for b in range(BH):
        for i in range(m):
            p = special.softmax(beta * Kn[b, :i + 1] @ Qn[b, i])
            np.testing.assert_allclose(O0[b, i], p @ Vn[b, :i + 1], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- recentring / temperature
def pin_recentring_and_temperature(o):
    """Recentring and temperature (Sec. 2): with recenter off and tau = 1 the
    options change nothing; the pivots with temperature tau are those of the
    plain method on keys K / tau (key kernel exp(beta<x,y>/tau^2)); the
    pivots with recentring are those of the plain method on K - mean(K)
    (numpy), also with several bins, whose keys share the mean of all n keys
    of their instance; full-rank bins stay exact attention with both options
    on."""
    Q, K, V = _rand(151, 2, 20, 48, 6, scale=1.2)
    beta = 0.4
    a = o.wildcat_forward_binned(Q, K, V, beta, 16, 2, seed=3)
    b = o.wildcat_forward_binned(Q, K, V, beta, 16, 2, seed=3, recenter=False, tau=1.0)
    np.testing.assert_array_equal(a[0], b[0])
    tau = 1.7
    _, S_t, _ = o.wildcat_forward_binned(Q, K, V, beta, 16, 1, seed=4, tau=tau)
    _, S_k, _ = o.wildcat_forward(Q, K / tau, V, beta, 16, seed=4)
    np.testing.assert_array_equal(S_t, S_k)
    Kc = K - K.mean(axis=1, keepdims=True)
    _, S_r, _ = o.wildcat_forward_binned(Q, K, V, beta, 16, 1, seed=5, recenter=True)
    _, S_c, _ = o.wildcat_forward(Q, Kc, V, beta, 16, seed=5)
    np.testing.assert_array_equal(S_r, S_c)
    # bins: the instance's mean, not a bin's (bins drift apart so the means differ)
    Kd = K + 2.0 * (np.arange(K.shape[1]) // (K.shape[1] // 4))[None, :, None]
    Kdc = Kd - Kd.mean(axis=1, keepdims=True)
    _, S_rb, rk_rb = o.wildcat_forward_binned(Q, Kd, V, beta, 16, 4, seed=8, recenter=True)
    _, S_cb, rk_cb = o.wildcat_forward_binned(Q, Kdc, V, beta, 16, 4, seed=8)
    np.testing.assert_array_equal(S_rb, S_cb)
    np.testing.assert_array_equal(rk_rb, rk_cb)
    O, _, rank = o.wildcat_forward_binned(Q, K, V, beta, 48, 4, seed=6, eps=1e-14, recenter=True,
                                          tau=1.3)
    assert np.all(rank == 12)
    np.testing.assert_allclose(O, o.exact_attention(Q, K, V, beta), rtol=0, atol=1e-11)


# --------------------------------------------------------------------------- inverse route
def pin_inverse_route_weights(o):
    """The inverse-maintenance weights route equals a dense LU solve of
    h(K_S,K_S) X = h(K_S,K) (V,1) (numpy.linalg.solve) and the factor route on
    the same pivots; it interpolates (W[:, S] = I, checked through V = e_S
    columns); one pivot gives the closed form W = h(k_s, K) / h(k_s, k_s)."""
    n, d, r, beta = 44, 6, 10, 0.35
    _, K, V = _rand(161, 2, 1, n, d)
    res = o.rpcholesky(K, beta, r, seed=9, eps=1e-13)
    VS_f, w_f = o.weights(res["F"], res["S"], res["rank"], V)
    VS_i, w_i = o.weights_inverse(K, res["S"], res["rank"], V, beta)
    for b in range(2):
        rr = res["rank"][b]
        s = res["S"][b][:rr]
        H = _H(K[b], beta)
        ref = np.linalg.solve(H[np.ix_(s, s)], H[s, :]) @ np.concatenate([V[b], np.ones((n, 1))], 1)
        got = np.concatenate([VS_i[b][:rr], w_i[b][:rr, None]], 1)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-9 * np.abs(ref).max())
        np.testing.assert_allclose(VS_i[b], VS_f[b], rtol=0, atol=1e-9 * np.abs(VS_f[b]).max())
        np.testing.assert_allclose(w_i[b], w_f[b], rtol=0, atol=1e-9 * np.abs(w_f[b]).max())
        # interpolation: value column a = e_{S_a} (a < d) gives row a' weight delta_{a a'}
        E = np.zeros((1, n, d))
        E[0, s[:d], np.arange(d)] = 1.0
        VS_e, _ = o.weights_inverse(K[b:b + 1], res["S"][b:b + 1], res["rank"][b:b + 1], E, beta)
        np.testing.assert_allclose(VS_e[0][:rr], np.eye(rr, d), rtol=0, atol=1e-9)
    S1 = np.array([[7], [30]], np.int32)
    VS1, w1 = o.weights_inverse(K, S1, np.array([1, 1], np.int32), V, beta)
    for b in range(2):
        hk = np.exp(beta * (K[b] @ K[b][S1[b, 0]]))
        hkk = np.exp(beta * K[b][S1[b, 0]] @ K[b][S1[b, 0]])
        np.testing.assert_allclose(VS1[b, 0], hk @ V[b] / hkk, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(w1[b, 0], hk.sum() / hkk, rtol=1e-12)


ALL_PINS = [
    pin_exact_bruteforce,
    pin_full_rank_is_exact,
    pin_weights_textbook_solve,
    pin_inverse_update_route,
    pin_inverse_route_weights,
    pin_partial_cholesky_interpolates,
    pin_residual_invariants,
    pin_philox_matches_library,
    pin_uniform_mapping_matches_library,
    pin_uniforms_uniform,
    pin_first_pivot_law,
    pin_shift_invariance,
    pin_value_range_and_recentring,
    pin_error_falls_with_rank,
    pin_single_pivot_closed_form,
    pin_hand_examples,
    pin_binning_closed_forms,
    pin_binning_composes_unbinned_parts,
    pin_decode_closed_form,
    pin_recentring_and_temperature,
]
