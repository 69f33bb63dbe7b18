"""wildcat_attend_noalloc: the attend variant for callers that cannot
allocate device memory (they only hold pointers another component handed
them, or cannot afford a cudaMalloc in their loop), so they cannot pass the
workspace that wildcat_attend takes.  Its scratch is a static 1 MiB device
array inside the library.

Checked through the C ABI on two calls in a row with different shapes and
dtypes (the second call reuses the array the first one wrote): against the
fp64 oracle's attend on the same coreset at 1e-4 of the value range for both
dtypes (the no-alloc variant runs the float32 CUDA-core kernel), and against
wildcat_attend on the same inputs at the parity tolerance of the tests.  Plus
the host-side size limit.  This file is collected last so that a run stopping
at the first failure has already run every other test; it also passes alone
in a fresh process."""
import ctypes
import math

import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads

pytestmark = pytest.mark.gpu


def _coreset(dist, BH, n, m, d, r, dtype, seed):
    w = workloads.Workload(name="noalloc", B=BH, H=1, n=n, m=m, d=d, r=r, dtype=dtype, dist=dist,
                           beta=1.0 / math.sqrt(d), seed=seed, pivot_seed=seed + 1)
    dev, _ = workloads.make(w)
    Q, K, V = (dev[k].cuda() for k in ("Q", "K", "V"))
    S, F, rank, K_S = wc.select(K, w.beta, r, w.pivot_seed)
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, V)
    return w, (Q, K_S, rank, w.beta, V_S, wv, vmin, vmax)


def _np64(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_noalloc_matches_attend_on_two_calls():
    import oracle

    orc = oracle.get()
    calls = [
        _coreset("mixture16", 4, 784, 784, 64, 64, "bf16", 21),
        _coreset("iid", 3, 1000, 2333, 32, 40, "f32", 22),
    ]
    for w, args in calls:
        O_ref = wc.attend(*args)
        O_na = wc.attend_noalloc(*args)
        torch.cuda.synchronize()
        Q, K_S, rank, beta, V_S, wv, vmin, vmax = args
        lo, hi = _np64(vmin), _np64(vmax)
        span = np.maximum(hi - lo, 1e-30)[:, None, :]
        # the oracle's attend on exactly the coreset the device holds
        O_orc = orc.attend(_np64(Q), _np64(K_S), _np64(V_S), _np64(wv), rank.cpu().numpy(), lo, hi, beta)
        err_orc = np.max(np.abs(O_na.cpu().numpy() - O_orc) / span)
        assert err_orc <= 1e-4, (w.dtype, err_orc)
        # and wildcat_attend at the parity tolerance of the tests: 1e-4 of the value
        # range for float32 inputs, 2e-2 for bfloat16 (bf16 runs on the tensor cores)
        err = np.max(np.abs(O_na.cpu().numpy() - O_ref.cpu().numpy()) / span)
        assert err <= (1e-4 if w.dtype == "f32" else 2e-2), (w.dtype, err)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    L = wc.lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    BH, m = 8000, 1 << 20  # needs about 4 * 8000 * 65 bytes > 1 MiB
    st = L.wildcat_attend_noalloc(fake, fake, 1, BH, m, 64, 16, fake, 0.125, fake, fake, fake,
                                  fake, fake, None)
    assert st == 2
    assert b"1 MiB" in L.wildcat_last_error()
