"""wildcat_forward_binned (divide-and-conquer binning, Sec. 2) against the
oracle's binned forward, through the C ABI."""
import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

EPS = 1e-6


def test_one_bin_is_the_plain_forward():
    w = gc.case("bins1", "mixture16", 3, 1024, 1024, 64, 64, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 5)
    Ob, Sb, rb = wc.forward_binned(d["Q"], d["K"], d["V"], w.beta, w.r, 1, 5)
    assert torch.equal(Sb, S) and torch.equal(rb[:, 0], rank) and torch.equal(Ob, O)


@pytest.mark.parametrize("w,nbins", [
    (gc.case("bins_f32", "iid", 2, 2048, 300, 64, 64, "f32"), 4),
    (gc.case("bins_bf16", "normclip", 3, 4096, 500, 64, 128, "bf16"), 8),
    (gc.case("bins_d128", "iid", 2, 8192, 257, 128, 256, "bf16"), 16),
], ids=lambda x: x if isinstance(x, int) else x.name)
def test_binned_parity(orc, w, nbins):
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward_binned(d["Q"], d["K"], d["V"], w.beta, w.r, nbins, w.pivot_seed, EPS)
    assert wc.device_status() == 0
    O, S, rank = O.cpu().numpy(), S.cpu().numpy(), rank.cpu().numpy()
    nb, rb = w.n // nbins, w.r // nbins
    for b in range(w.BH):
        for q in range(nbins):
            rows = S[b, q * rb:q * rb + rank[b, q]]
            assert np.all((rows >= q * nb) & (rows < (q + 1) * nb))
            assert np.all(S[b, q * rb + rank[b, q]:(q + 1) * rb] == -1)
        valid = S[b][S[b] >= 0]
        assert len(set(valid.tolist())) == len(valid)
    # the oracle on the device's pivots (and stopping steps)
    O_o, S_o, rank_o = orc.wildcat_forward_binned(ex["Q"], ex["K"], ex["V"], w.beta, w.r, nbins,
                                                  eps=0.0, S_fixed=S)
    assert np.array_equal(S_o, S) and np.array_equal(rank_o, rank)
    lo, hi = orc.value_range(ex["V"])
    assert np.all(O >= lo[:, None, :]) and np.all(O <= hi[:, None, :])
    assert gc.r12(O, O_o, lo, hi) <= gc.TOL_R12[w.dtype]
    # the oracle's own draws agree step by step until a near-tie (bin by bin)
    gc.binned_pivots_agree_until_tie(orc, ex["K"], w.beta, w.r, nbins, w.pivot_seed, EPS, S, rank)


def test_full_rank_bins_recover_exact_attention(orc):
    w = gc.case("bins_full", "iid", 2, 96, 40, 32, 96, "f32", beta=0.25)
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward_binned(d["Q"], d["K"], d["V"], w.beta, w.r, 4, 1, 1e-7)
    assert rank.cpu().numpy().tolist() == [[24] * 4] * 2
    Oe = orc.exact_attention(ex["Q"], ex["K"], ex["V"], w.beta)
    lo, hi = orc.value_range(ex["V"])
    assert gc.r12(O.cpu().numpy(), Oe, lo, hi) <= 1e-4


def test_binned_rejects_uneven_bins():
    import ctypes

    L = wc.lib()
    fake = ctypes.c_void_p(1 << 20)
    assert L.wildcat_forward_binned(fake, fake, fake, 1, 2, 10, 1000, 64, 0.125, 64, 3, 0, 0, 1e-6,
                                    fake, None, None, fake, 1 << 30, None) == 1
    assert L.wildcat_forward_binned_workspace_size(2, 10, 1000, 64, 60, 7, 1) == 0
