"""wildcat_decode_attend (KV-cache decode with new tokens, Sec. 2) against
the oracle, through the C ABI: new tokens attend over the compressed cache
and causally over themselves."""
import math

import numpy as np
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


def _compressed_cache(w):
    dev, ex = workloads.make(w)
    d = gc.cuda_inputs(dev)
    S, F, rank, K_S = wc.select(d["K"], w.beta, w.r, w.pivot_seed)
    V_S, wv, vmin, vmax = wc.weights(F, S, rank, d["V"])
    return dev, ex, d, (K_S, rank, V_S, wv, vmin, vmax)


@pytest.mark.parametrize("w,m", [
    (gc.case("dec_kv", "walk", 4, 8192, 64, 128, 256, "bf16"), 64),
    (gc.case("dec_ragged", "iid", 3, 3000, 10, 64, 96, "f32"), 77),
    (gc.case("dec_d32", "normclip", 2, 2048, 10, 32, 64, "bf16"), 130),
], ids=lambda x: x if isinstance(x, int) else x.name)
def test_decode_parity(orc, w, m):
    dev, ex, d, (K_S, rank, V_S, wv, vmin, vmax) = _compressed_cache(w)
    rng = np.random.default_rng(5)
    new = {k: workloads.round_to(rng.standard_normal((w.BH, m, w.d)), w.dtype) for k in "QKV"}
    O = wc.decode_attend(new["Q"][0].cuda(), new["K"][0].cuda(), new["V"][0].cuda(), K_S, rank,
                         w.beta, V_S, wv, vmin, vmax).cpu().numpy()
    O_o = orc.decode_attend(new["Q"][1], new["K"][1], new["V"][1],
                            K_S.float().cpu().numpy().astype(np.float64),
                            V_S.cpu().numpy().astype(np.float64), wv.cpu().numpy().astype(np.float64),
                            rank.cpu().numpy(), vmin.cpu().numpy().astype(np.float64),
                            vmax.cpu().numpy().astype(np.float64), w.beta)
    lo = np.minimum(vmin.cpu().numpy(), new["V"][1].min(1))
    hi = np.maximum(vmax.cpu().numpy(), new["V"][1].max(1))
    assert np.all(O >= lo[:, None, :]) and np.all(O <= hi[:, None, :])
    assert gc.r12(O, O_o, lo, hi) <= 1e-4


def test_decode_full_rank_cache_is_exact_causal_attention(orc):
    """Cache compressed at r = n: decode equals exact causal attention over
    the cached keys plus the new keys j <= i."""
    w = gc.case("dec_full", "iid", 2, 40, 10, 32, 40, "f32", beta=0.25)
    dev, ex, d, (K_S, rank, V_S, wv, vmin, vmax) = _compressed_cache(w)
    assert rank.cpu().tolist() == [40, 40]
    rng = np.random.default_rng(9)
    m = 9
    Qn, Kn, Vn = (rng.standard_normal((2, m, 32)).astype(np.float32) for _ in range(3))
    O = wc.decode_attend(*(torch.from_numpy(x).cuda() for x in (Qn, Kn, Vn)), K_S, rank, w.beta,
                         V_S, wv, vmin, vmax).cpu().numpy()
    for b in range(2):
        for i in range(m):
            keys = np.concatenate([ex["K"][b], Kn[b, :i + 1]])
            vals = np.concatenate([ex["V"][b], Vn[b, :i + 1]])
            s = w.beta * keys @ Qn[b, i].astype(np.float64)
            p = np.exp(s - s.max())
            ref = p @ vals / p.sum()
            span = np.maximum(vals.max(0) - vals.min(0), 1e-30)
            assert np.max(np.abs(O[b, i] - ref) / span) <= 1e-4
