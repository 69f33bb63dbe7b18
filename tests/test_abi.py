"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/wildcat.h declares, and rejects bad arguments on the host before any
CUDA call.  No compute call is made here."""
import ctypes

import pytest

import nystr_coreset_approximate_b200 as wc

FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first


@pytest.fixture(scope="module")
def L():
    return wc.lib()


def test_exports_every_declared_symbol(L):
    names = wc.declared_symbols()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert set(names) == set(wc._SIGS), "binding signatures out of sync with the header"


def test_status_strings_and_version(L):
    assert L.wildcat_version() >= 100
    assert L.wildcat_status_string(0) == b"WILDCAT_OK"
    assert L.wildcat_status_string(4) == b"WILDCAT_ERR_WORKSPACE"
    assert L.wildcat_status_string(99) == b"WILDCAT_UNKNOWN_STATUS"


def _select(L, **kw):
    a = dict(K=FAKE, dtype=1, BH=2, n=100, d=64, beta=0.125, r=10, seed=0, inst0=0, eps=1e-6, S=FAKE,
             F=FAKE, rank=FAKE, K_S=None, stream=None)
    a.update(kw)
    return L.wildcat_select(a["K"], a["dtype"], a["BH"], a["n"], a["d"], a["beta"], a["r"], a["seed"],
                            a["inst0"], a["eps"], a["S"], a["F"], a["rank"], a["K_S"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), 1),
    (dict(r=0), 1),
    (dict(r=101), 1),
    (dict(n=0), 1),
    (dict(BH=-1), 1),
    (dict(d=48), 2),
    (dict(d=256), 2),
    (dict(beta=float("nan")), 1),
    (dict(beta=-1.0), 1),
    (dict(eps=-1.0), 1),
    (dict(K=None), 1),
    (dict(F=None), 1),
    (dict(S=None), 1),
    (dict(K=ctypes.c_void_p((1 << 20) + 4)), 1),  # misaligned
    (dict(r=9000, n=10000), 2),
    (dict(inst0=-1), 1),
    (dict(inst0=2**32 - 1), 1),
])
def test_select_rejects_on_host(L, kw, code):
    assert _select(L, **kw) == code
    assert L.wildcat_last_error() != b""


def test_empty_batch_is_a_no_op(L):
    assert _select(L, BH=0, K=None, F=None, S=None, rank=None) == 0


def test_weights_and_attend_reject_on_host(L):
    ws = int(L.wildcat_weights_workspace_size(2, 100, 64, 10))
    assert ws > 0
    # workspace too small
    assert L.wildcat_weights(FAKE, FAKE, FAKE, FAKE, 1, 2, 100, 64, 10, FAKE, FAKE, FAKE, FAKE,
                             ctypes.c_void_p(1 << 20), 16, None) == 4
    # misaligned workspace
    assert L.wildcat_weights(FAKE, FAKE, FAKE, FAKE, 1, 2, 100, 64, 10, FAKE, FAKE, FAKE, FAKE,
                             ctypes.c_void_p((1 << 20) + 64), ws, None) == 4
    assert L.wildcat_attend(FAKE, FAKE, 1, 2, 50, 64, 10, FAKE, -0.5, FAKE, FAKE, FAKE, FAKE,
                            FAKE, FAKE, 1 << 20, None) == 1
    assert L.wildcat_attend(None, FAKE, 1, 2, 50, 64, 10, FAKE, 0.5, FAKE, FAKE, FAKE, FAKE,
                            FAKE, FAKE, 1 << 20, None) == 1


def test_forward_workspace_accounts_for_the_factor(L):
    BH, m, n, d, r = 32, 3136, 3136, 64, 128
    ws = int(L.wildcat_forward_workspace_size(BH, m, n, d, r, 1))
    assert ws >= 4 * BH * r * n  # F [BH, r, n] float32 lives in the workspace
    assert ws < 4 * BH * r * n * 2
    wh = int(L.wildcat_forward_host_workspace_size(BH, m, n, d, r, 1))
    assert wh >= ws + 2 * BH * (m + 2 * n) * d + 4 * BH * m * d
    assert L.wildcat_forward(FAKE, FAKE, FAKE, 1, BH, m, n, d, 0.125, r, 0, 0, 1e-6, FAKE, None,
                             None, ctypes.c_void_p(1 << 20), ws - 4096, None) == 4


def test_forward_ex_host_workspace_and_checks(L):
    BH, m, n, d, r = 8, 1024, 4096, 128, 64
    opts = wc.Options(4, 1, 1.5)
    we = int(L.wildcat_forward_ex_workspace_size(BH, m, n, d, r, 1, ctypes.byref(opts)))
    wh = int(L.wildcat_forward_ex_host_workspace_size(BH, m, n, d, r, 1, ctypes.byref(opts)))
    # the device forward's workspace plus staging for Q, K, V, O, S and the bins' ranks
    assert wh >= we + 2 * BH * (m + 2 * n) * d + 4 * BH * m * d + 4 * BH * r + 4 * BH * 4
    assert int(L.wildcat_forward_ex_host_workspace_size(BH, m, n, d, r, 1, ctypes.byref(wc.Options(3, 0, 1.0)))) == 0
    # rejected before any copy: bins that do not divide n, a bad temperature, a null input
    for o in (wc.Options(3, 0, 1.0), wc.Options(1, 0, 0.0)):
        assert L.wildcat_forward_ex_host(FAKE, FAKE, FAKE, 1, BH, m, n, d, 0.125, r, 0, 0, 1e-6,
                                         ctypes.byref(o), FAKE, None, None, FAKE, 1 << 30, None) == 1
    assert L.wildcat_forward_ex_host(FAKE, None, FAKE, 1, BH, m, n, d, 0.125, r, 0, 0, 1e-6,
                                     None, FAKE, None, None, FAKE, 1 << 30, None) == 1


def test_cluster_knob_validation(L):
    assert L.wildcat_set_select_cluster(3) == 1
    assert L.wildcat_set_select_cluster(32) == 1
    assert L.wildcat_set_select_cluster(4) == 0
    assert L.wildcat_set_select_cluster(0) == 0


def test_select_kernel_and_phase_knobs(L):
    """The select knobs validate on the host; the per-thread records read 0
    before any select call."""
    try:
        for bad in (-1, 2, 4, 5, 99):
            assert L.wildcat_set_select_kernel(bad) == 1
        for k in (0, 1, 3):
            assert L.wildcat_set_select_kernel(k) == 0
        for steps in (-1, 0, 16, 64):
            assert L.wildcat_set_select_phase_steps(steps) == 0
        assert L.wildcat_last_select_kernel() == 0
        assert L.wildcat_last_select_threads() == 0
        assert L.wildcat_last_select_phases() == 0
        assert L.wildcat_set_stage_events(None, None) == 0
    finally:
        L.wildcat_set_select_kernel(0)
        L.wildcat_set_select_phase_steps(0)


def test_select_workspace_holds_the_phase_state(L):
    """The select workspace carries two residual copies per instance for the
    global-sync exchange and one for a paused phase: at least 3 * 4 * BH * n
    bytes, and it grows linearly with BH * n."""
    for BH, n in ((32, 32768), (8, 131072), (1, 1024)):
        ws = int(L.wildcat_select_workspace_size(BH, n))
        assert ws >= 3 * 4 * BH * n
    a = int(L.wildcat_select_workspace_size(8, 16384))
    b = int(L.wildcat_select_workspace_size(8, 32768))
    assert 3 * 4 * 8 * 16384 <= b - a <= 4 * 4 * 8 * 16384


def test_binding_fails_loudly_without_cuda_tensors():
    import torch

    K = torch.zeros(1, 8, 64)
    with pytest.raises(ValueError):
        wc.select(K, 0.1, 2, out=(torch.zeros(1, 2, dtype=torch.int32), torch.zeros(1, 2, 8),
                                   torch.zeros(1, dtype=torch.int32), None))
