"""Seeded synthetic workloads for the WildCat hot path.

This module only draws inputs; it holds none of the method's arithmetic.
It is the one piece shared by the tests, the benchmark and the CPU oracle's
callers.  The shapes stand in for the workloads of "WildCat: Near-Linear
Attention in Theory and Practice" (Sec. 5 experiments: T2T-ViT image
classification, BigGAN image generation, Qwen2.5 KV-cache compression, and
the sequence-length sweep against FlashAttention-2).  None of those datasets
or weights is available; every tensor here is seeded Gaussian data with the
stated structure.

Recipe (all draws in float64 from ``numpy.random.default_rng(seed)``, then
rounded to the input dtype with round-to-nearest-even):

  iid        Q, K, V entries i.i.d. N(0, 1)                       (drawn in that order)
  mixture16  per instance 16 centres ~ N(0, I_d); key = centre (uniform choice)
             + 0.3 N(0, I); query = key + 0.1 N(0, I); V ~ N(0, 1)
  normclip   Q, K ~ N(0, I), each row x <- x * min(1, sqrt(d) / |x|); V ~ N(0, 1)
  walk       K and V: x_l = mu_l + N(0, I), mu_0 = 0, mu_l = mu_{l-1} + 0.01 N(0, I)
             (separate walks for K and V, per head); Q ~ N(0, 1)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    n: int
    m: int
    d: int
    r: int
    dtype: str          # "f32" or "bf16"
    dist: str           # iid | mixture16 | normclip | walk
    beta: float
    seed: int           # numpy seed of the inputs
    pivot_seed: int     # Philox key of the pivot draws

    @property
    def BH(self) -> int:
        return self.B * self.H

    def scaled(self, **kw) -> "Workload":
        """Same distribution at other sizes (for parity tests)."""
        return replace(self, **kw)


def _cfg(c, name, B, H, n, m, d, r, dtype, dist):
    return Workload(name=name, B=B, H=H, n=n, m=m, d=d, r=r, dtype=dtype, dist=dist,
                    beta=1.0 / math.sqrt(d), seed=1000 + c, pivot_seed=c)


#: The five workload families (config 4 has three sequence lengths).
CONFIGS: Dict[str, Workload] = {
    "c0_unit": _cfg(0, "c0_unit", 1, 1, 1024, 1024, 64, 32, "f32", "iid"),
    "c1_vit56": _cfg(1, "c1_vit56", 32, 1, 3136, 3136, 64, 128, "bf16", "mixture16"),
    "c2_imggen64": _cfg(2, "c2_imggen64", 8, 16, 4096, 4096, 64, 256, "bf16", "normclip"),
    "c3_kvcache": _cfg(3, "c3_kvcache", 1, 32, 32768, 64, 128, 1024, "bf16", "walk"),
    "c4a_long16k": _cfg(4, "c4a_long16k", 1, 8, 16384, 16384, 128, 512, "bf16", "iid"),
    "c4b_long64k": _cfg(4, "c4b_long64k", 1, 8, 65536, 65536, 128, 512, "bf16", "iid"),
    "c4c_long128k": _cfg(4, "c4c_long128k", 1, 8, 131072, 131072, 128, 512, "bf16", "iid"),
}


def _rowclip(x: np.ndarray) -> np.ndarray:
    d = x.shape[-1]
    nrm = np.linalg.norm(x, axis=-1, keepdims=True)
    return x * np.minimum(1.0, math.sqrt(d) / np.maximum(nrm, 1e-300))


def generate(w: Workload) -> Dict[str, np.ndarray]:
    """Draw Q [BH, m, d], K [BH, n, d], V [BH, n, d] in float64 (not yet rounded)."""
    rng = np.random.default_rng(w.seed)
    BH, n, m, d = w.BH, w.n, w.m, w.d
    if w.dist == "iid":
        Q = rng.standard_normal((BH, m, d))
        K = rng.standard_normal((BH, n, d))
        V = rng.standard_normal((BH, n, d))
    elif w.dist == "mixture16":
        if m != n:
            raise ValueError("mixture16 draws one query per key (m == n)")
        centres = rng.standard_normal((BH, 16, d))
        choice = rng.integers(0, 16, size=(BH, n))
        K = np.take_along_axis(centres, choice[..., None], axis=1) \
            + 0.3 * rng.standard_normal((BH, n, d))
        Q = K + 0.1 * rng.standard_normal((BH, n, d))
        V = rng.standard_normal((BH, n, d))
    elif w.dist == "normclip":
        Q = _rowclip(rng.standard_normal((BH, m, d)))
        K = _rowclip(rng.standard_normal((BH, n, d)))
        V = rng.standard_normal((BH, n, d))
    elif w.dist == "walk":
        stepK = 0.01 * rng.standard_normal((BH, n, d))
        stepK[:, 0, :] = 0.0
        K = np.cumsum(stepK, axis=1) + rng.standard_normal((BH, n, d))
        stepV = 0.01 * rng.standard_normal((BH, n, d))
        stepV[:, 0, :] = 0.0
        V = np.cumsum(stepV, axis=1) + rng.standard_normal((BH, n, d))
        Q = rng.standard_normal((BH, m, d))
    else:
        raise ValueError(f"unknown distribution {w.dist!r}")
    return {"Q": Q, "K": K, "V": V}


def round_to(x: np.ndarray, dtype: str):
    """Round float64 data to the input dtype (round-to-nearest-even).

    Returns (torch CPU tensor in that dtype, float64 numpy copy of exactly the
    rounded values).  The oracle consumes the second, the device the first.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "f32":
        t = t.to(torch.float32)
    elif dtype == "bf16":
        t = t.to(torch.float32).to(torch.bfloat16)
    else:
        raise ValueError(dtype)
    return t.contiguous(), t.to(torch.float64).numpy()


def make(w: Workload):
    """Generate and round a workload.  Returns (device-ready CPU tensors,
    float64 exact copies) as two dicts keyed Q, K, V."""
    raw = generate(w)
    dev, exact = {}, {}
    for k, v in raw.items():
        dev[k], exact[k] = round_to(v, w.dtype)
    return dev, exact


def sample_rows(w: Workload, count: int = 256) -> np.ndarray:
    """Seeded query rows used where the oracle cannot afford every row."""
    rng = np.random.default_rng(w.seed + 7919)
    count = min(count, w.m)
    return np.sort(rng.choice(w.m, size=count, replace=False)).astype(np.int64)
