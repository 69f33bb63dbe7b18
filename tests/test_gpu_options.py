"""wildcat_forward_ex (bins, key recentring, temperature; Sec. 2) against the
oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

EPS = 1e-6


def test_default_options_are_the_plain_forward():
    w = gc.case("opt_default", "mixture16", 3, 1024, 1024, 64, 64, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward(d["Q"], d["K"], d["V"], w.beta, w.r, 5)
    Oe, Se, re = wc.forward_ex(d["Q"], d["K"], d["V"], w.beta, w.r, 5)
    assert torch.equal(Se, S) and torch.equal(re[:, 0], rank) and torch.equal(Oe, O)


@pytest.mark.parametrize("w,nbins,recenter,tau", [
    (gc.case("opt_walk_rc", "walk", 2, 4096, 64, 128, 128, "bf16"), 1, True, 1.0),
    (gc.case("opt_walk_all", "walk", 2, 4096, 64, 128, 128, "bf16"), 4, True, 1.6),
    (gc.case("opt_tau_f32", "iid", 2, 2000, 300, 64, 50, "f32"), 2, False, 2.0),
    (gc.case("opt_rc_f32", "normclip", 3, 1024, 100, 32, 32, "f32"), 1, True, 1.0),
], ids=lambda x: x.name if hasattr(x, "name") else str(x))
def test_options_parity(orc, w, nbins, recenter, tau):
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O, S, rank = wc.forward_ex(d["Q"], d["K"], d["V"], w.beta, w.r, w.pivot_seed, EPS, nbins=nbins,
                               recenter=recenter, tau=tau)
    assert wc.device_status() == 0
    O, S, rank = O.cpu().numpy(), S.cpu().numpy(), rank.cpu().numpy()
    O_o, S_o, rank_o = orc.wildcat_forward_binned(ex["Q"], ex["K"], ex["V"], w.beta, w.r, nbins,
                                                  eps=0.0, S_fixed=S, recenter=recenter, tau=tau)
    assert np.array_equal(S_o, S) and np.array_equal(rank_o, rank)
    lo, hi = orc.value_range(ex["V"])
    assert np.all(O >= lo[:, None, :]) and np.all(O <= hi[:, None, :])
    assert gc.r12(O, O_o, lo, hi) <= gc.TOL_R12[w.dtype]
    # the oracle's own draws agree step by step until a near-tie (bin by bin)
    gc.binned_pivots_agree_until_tie(orc, ex["K"], w.beta, w.r, nbins, w.pivot_seed, EPS, S, rank,
                                     recenter=recenter, tau=tau)


@pytest.mark.parametrize("nbins,recenter,tau", [(4, False, 1.0), (2, True, 1.6), (1, False, 1.0)])
def test_forward_ex_host_matches_device(nbins, recenter, tau):
    """The host-buffer extended forward (K copied first, V and Q while the
    select runs) gives the device forward's outputs bit for bit."""
    w = gc.case("ex_host", "walk", 3, 4096, 300, 128, 128, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    O_d, S_d, r_d = wc.forward_ex(d["Q"], d["K"], d["V"], w.beta, w.r, 11, EPS, nbins=nbins,
                                  recenter=recenter, tau=tau)
    pinned = {k: v.pin_memory() for k, v in dev.items()}
    O_h, S_h, r_h = wc.forward_ex_host(pinned["Q"], pinned["K"], pinned["V"], w.beta, w.r, 11, EPS,
                                       nbins=nbins, recenter=recenter, tau=tau)
    assert torch.equal(S_h, S_d.cpu()) and torch.equal(r_h, r_d.cpu()) and torch.equal(O_h, O_d.cpu())


def test_options_rejected_on_host():
    import ctypes

    L = wc.lib()
    fake = ctypes.c_void_p(1 << 20)
    for opts in (wc.Options(1, 2, 1.0), wc.Options(1, 0, 0.0), wc.Options(1, 0, float("nan")),
                 wc.Options(3, 0, 1.0)):
        assert L.wildcat_forward_ex(fake, fake, fake, 1, 2, 10, 1024, 64, 0.125, 64, 0, 0, 1e-6,
                                    ctypes.byref(opts), fake, None, None, fake, 1 << 30, None) == 1
