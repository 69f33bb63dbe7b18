"""fp64 CPU oracle for the WildCat hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
and its binding) never imports it, and it never imports the product.

The arithmetic lives in ``wildcat_oracle.c`` (plain C, double precision,
sequential sums); this module only compiles it with gcc and marshals numpy
arrays through ctypes.  Each function names the part of "WildCat:
Near-Linear Attention in Theory and Practice" (Sec. 2) that it follows.

Array conventions: Q [BH, m, d], K and V [BH, n, d], all float64, C order.
The factor F is [BH, r, n] (column i of the n x r factor is contiguous).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wildcat_oracle.c")
_LIB_NAME = "liboracle.so"

_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u32p = ctypes.POINTER(ctypes.c_uint32)


def build(out_path: Optional[str] = None, mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle into a shared library (gcc, OpenMP, no fast-math)."""
    if out_path is None:
        out_path = os.path.join(_HERE, _LIB_NAME)
    if (not force and mutant == 0 and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(_SRC)):
        return out_path
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-shared", "-fPIC", f"-DORACLE_MUTANT={int(mutant)}", "-o", out_path, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out_path


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    lib.oracle_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
    lib.oracle_philox4x32_10.restype = None
    lib.oracle_pivot_uniform.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64]
    lib.oracle_pivot_uniform.restype = ctypes.c_double
    lib.oracle_pivot_uniforms.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, _f64p]
    lib.oracle_pivot_uniforms.restype = None
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_exact_attention.argtypes = [_f64p, _f64p, _f64p, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_int, ctypes.c_double, _i64p,
                                           ctypes.c_int64, _f64p]
    lib.oracle_exact_attention.restype = ctypes.c_int
    lib.oracle_rpcholesky.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_uint64,
                                      ctypes.c_double, ctypes.c_int, _i32p, _i32p, _f64p, _i32p,
                                      _f64p, _f64p]
    lib.oracle_rpcholesky.restype = ctypes.c_int
    lib.oracle_weights.argtypes = [_f64p, _i32p, _i32p, _f64p, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int, ctypes.c_int, _f64p, _f64p]
    lib.oracle_weights.restype = ctypes.c_int
    lib.oracle_weights_inverse.argtypes = [_f64p, _i32p, _i32p, _f64p, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_double, _f64p, _f64p]
    lib.oracle_weights_inverse.restype = ctypes.c_int
    lib.oracle_value_range.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                       _f64p, _f64p]
    lib.oracle_value_range.restype = None
    lib.oracle_gather.argtypes = [_f64p, _i32p, _i32p, ctypes.c_int64, ctypes.c_int64,
                                  ctypes.c_int, ctypes.c_int, _f64p]
    lib.oracle_gather.restype = None
    lib.oracle_attend.argtypes = [_f64p, _f64p, _f64p, _f64p, _i32p, _f64p, _f64p,
                                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_double, _i64p, ctypes.c_int64, _f64p]
    lib.oracle_attend.restype = ctypes.c_int
    lib.oracle_wildcat_forward.argtypes = [_f64p, _f64p, _f64p, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_int, ctypes.c_uint64, ctypes.c_double,
                                           _i32p, _i64p, ctypes.c_int64, _f64p, _i32p, _i32p]
    lib.oracle_wildcat_forward.restype = ctypes.c_int
    lib.oracle_wildcat_forward_binned.argtypes = [_f64p, _f64p, _f64p, ctypes.c_int64,
                                                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                                  ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_double,
                                                  ctypes.c_uint64, ctypes.c_double, _i32p, _i64p,
                                                  ctypes.c_int64, _f64p, _i32p, _i32p]
    lib.oracle_wildcat_forward_binned.restype = ctypes.c_int
    lib.oracle_decode_attend.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _i32p, _f64p,
                                         _f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_double, _f64p]
    lib.oracle_decode_attend.restype = ctypes.c_int
    return lib


class Oracle:
    """ctypes front end of one compiled oracle library (the real one or a mutant)."""

    def __init__(self, lib_path: Optional[str] = None):
        self.path = lib_path or build()
        self.lib = _declare(ctypes.CDLL(self.path))

    # -- helpers ---------------------------------------------------------------
    @staticmethod
    def _f64(a):
        a = np.ascontiguousarray(a, dtype=np.float64)
        return a, a.ctypes.data_as(_f64p)

    @staticmethod
    def _i32(a):
        if a is None:
            return None, None
        a = np.ascontiguousarray(a, dtype=np.int32)
        return a, a.ctypes.data_as(_i32p)

    @staticmethod
    def _rows(rows):
        if rows is None:
            return None, None, 0
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        return rows, rows.ctypes.data_as(_i64p), int(rows.shape[0])

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    # -- random stream ---------------------------------------------------------
    def philox4x32_10(self, ctr, key):
        """Philox4x32-10 block (Salmon et al., SC'11) for one counter and key."""
        c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
        k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
        o = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(c, k, o)
        return [int(x) for x in o]

    def pivot_uniform(self, seed: int, step: int, inst: int) -> float:
        """Uniform in (0, 1] that draws pivot `step` of instance `inst`."""
        return float(self.lib.oracle_pivot_uniform(int(seed), int(step), int(inst)))

    def pivot_uniforms(self, seed: int, BH: int, steps: int) -> np.ndarray:
        """u[b, i] for every instance b < BH and step i < steps."""
        u = np.zeros((BH, steps))
        self.lib.oracle_pivot_uniforms(int(seed), int(BH), int(steps), u.ctypes.data_as(_f64p))
        return u

    # -- exact attention ---------------------------------------------------------
    def exact_attention(self, Q, K, V, beta, rows=None):
        """O = D^-1 A V with A = exp(beta Q K^T) (Sec. 2, opening paragraph)."""
        Q, qp = self._f64(Q)
        K, kp = self._f64(K)
        V, vp = self._f64(V)
        BH, m, d = Q.shape
        n = K.shape[1]
        rows_a, rp, nr = self._rows(rows)
        O = np.zeros((BH, nr if rows is not None else m, d))
        err = self.lib.oracle_exact_attention(qp, kp, vp, BH, m, n, d, float(beta), rp, nr,
                                              O.ctypes.data_as(_f64p))
        if err:
            raise MemoryError("oracle_exact_attention")
        return O

    # -- RPCholesky select ----------------------------------------------------------
    def rpcholesky(self, K, beta, r, seed=0, eps=1e-6, shift=True, S_fixed=None,
                   history=False):
        """RPCholesky coreset selection with its partial Cholesky factor
        (Sec. 2, randomly pivoted Cholesky; Alg. 1 RPNys).

        Returns dict(S [BH,r] int32, F [BH,r,n], rank [BH], hist [BH,r+1,n]
        (history=True), margin [BH,r]).
        """
        K, kp = self._f64(K)
        BH, n, d = K.shape
        Sf, sfp = self._i32(S_fixed)
        S = np.full((BH, r), -1, dtype=np.int32)
        F = np.zeros((BH, r, n))
        rank = np.zeros(BH, dtype=np.int32)
        hist = np.zeros((BH, r + 1, n)) if history else None
        margin = np.full((BH, r), np.nan)
        err = self.lib.oracle_rpcholesky(
            kp, BH, n, d, float(beta), int(r), int(seed), float(eps), int(bool(shift)), sfp,
            S.ctypes.data_as(_i32p), F.ctypes.data_as(_f64p), rank.ctypes.data_as(_i32p),
            hist.ctypes.data_as(_f64p) if history else None, margin.ctypes.data_as(_f64p))
        if err:
            raise MemoryError("oracle_rpcholesky")
        return {"S": S, "F": F, "rank": rank, "hist": hist, "margin": margin}

    # -- weights -------------------------------------------------------------------
    def weights(self, F, S, rank, V):
        """W (V, 1_n) = F_S^-T F^T (V, 1_n): returns (V_S [BH,r,d], w [BH,r])
        (Sec. 2; Alg. 2 CompressKV, V_S = W V and w = W 1_n)."""
        F, fp = self._f64(F)
        S, sp = self._i32(S)
        rank, rkp = self._i32(rank)
        V, vp = self._f64(V)
        BH, r, n = F.shape
        d = V.shape[2]
        VS = np.zeros((BH, r, d))
        w = np.zeros((BH, r))
        err = self.lib.oracle_weights(fp, sp, rkp, vp, BH, n, d, r, VS.ctypes.data_as(_f64p),
                                      w.ctypes.data_as(_f64p))
        if err:
            raise MemoryError("oracle_weights")
        return VS, w

    def weights_inverse(self, K, S, rank, V, beta):
        """The same W (V, 1_n) through h(K_S, K_S)^-1 maintained by the rank-one
        update of RPNys (Sec. 2): returns (V_S [BH,r,d], w [BH,r])."""
        K, kp = self._f64(K)
        S, sp = self._i32(S)
        rank, rkp = self._i32(rank)
        V, vp = self._f64(V)
        BH, n, d = K.shape
        r = S.shape[1]
        VS = np.zeros((BH, r, d))
        w = np.zeros((BH, r))
        err = self.lib.oracle_weights_inverse(kp, sp, rkp, vp, BH, n, d, r, float(beta),
                                              VS.ctypes.data_as(_f64p), w.ctypes.data_as(_f64p))
        if err:
            raise MemoryError("oracle_weights_inverse")
        return VS, w

    def value_range(self, V):
        """Column-wise [v_min j, v_max j] of V per instance (Sec. 2, value-range clip)."""
        V, vp = self._f64(V)
        BH, n, d = V.shape
        vmin = np.zeros((BH, d))
        vmax = np.zeros((BH, d))
        self.lib.oracle_value_range(vp, BH, n, d, vmin.ctypes.data_as(_f64p),
                                    vmax.ctypes.data_as(_f64p))
        return vmin, vmax

    def gather(self, K, S, rank):
        """K_S = rows S of K, zero past the rank (Alg. 2 CompressKV)."""
        K, kp = self._f64(K)
        S, sp = self._i32(S)
        rank, rkp = self._i32(rank)
        BH, n, d = K.shape
        r = S.shape[1]
        KS = np.zeros((BH, r, d))
        self.lib.oracle_gather(kp, sp, rkp, BH, n, d, r, KS.ctypes.data_as(_f64p))
        return KS

    # -- weighted attend --------------------------------------------------------------
    def attend(self, Q, KS, VS, w, rank, vmin, vmax, beta, rows=None):
        """O_hat = clip(diag(U w)^-1 U V_S), U = exp(beta Q K_S^T - beta M_Q)
        (Sec. 2 plug-in estimator and value-range clip; Alg. 3 WtdAttn)."""
        Q, qp = self._f64(Q)
        KS, ksp = self._f64(KS)
        VS, vsp = self._f64(VS)
        w, wp = self._f64(w)
        rank, rkp = self._i32(rank)
        vmin, lop = self._f64(vmin)
        vmax, hip = self._f64(vmax)
        BH, m, d = Q.shape
        r = KS.shape[1]
        rows_a, rp, nr = self._rows(rows)
        O = np.zeros((BH, nr if rows is not None else m, d))
        err = self.lib.oracle_attend(qp, ksp, vsp, wp, rkp, lop, hip, BH, m, d, r, float(beta),
                                     rp, nr, O.ctypes.data_as(_f64p))
        if err:
            raise MemoryError("oracle_attend")
        return O

    # -- whole forward -----------------------------------------------------------------
    def wildcat_forward(self, Q, K, V, beta, r, seed=0, eps=1e-6, S_fixed=None, rows=None):
        """WildCat module (Alg. 4): CompressKV then WtdAttn.  Returns (O_hat, S, rank)."""
        Q, qp = self._f64(Q)
        K, kp = self._f64(K)
        V, vp = self._f64(V)
        BH, m, d = Q.shape
        n = K.shape[1]
        Sf, sfp = self._i32(S_fixed)
        rows_a, rp, nr = self._rows(rows)
        O = np.zeros((BH, nr if rows is not None else m, d))
        S = np.full((BH, r), -1, dtype=np.int32)
        rank = np.zeros(BH, dtype=np.int32)
        err = self.lib.oracle_wildcat_forward(qp, kp, vp, BH, m, n, d, float(beta), int(r),
                                              int(seed), float(eps), sfp, rp, nr,
                                              O.ctypes.data_as(_f64p), S.ctypes.data_as(_i32p),
                                              rank.ctypes.data_as(_i32p))
        if err:
            raise MemoryError("oracle_wildcat_forward")
        return O, S, rank


    def wildcat_forward_binned(self, Q, K, V, beta, r, nbins, seed=0, eps=1e-6, rows=None,
                               S_fixed=None, recenter=False, tau=1.0):
        """WildCat with divide-and-conquer binning (Sec. 2): nbins contiguous
        bins, r / nbins pivots each, block-diagonal weights, attend over the
        union; optionally on recentred keys and with temperature tau (key
        kernel exp(beta <x,y> / tau^2)).  Returns (O_hat, S [BH, r] global
        key indices, rank [BH, nbins])."""
        Q, qp = self._f64(Q)
        K, kp = self._f64(K)
        V, vp = self._f64(V)
        BH, m, d = Q.shape
        n = K.shape[1]
        rows_a, rp, nr = self._rows(rows)
        O = np.zeros((BH, nr if rows is not None else m, d))
        S = np.full((BH, r), -1, dtype=np.int32)
        rank = np.zeros((BH, nbins), dtype=np.int32)
        Sf, sfp = self._i32(S_fixed)
        err = self.lib.oracle_wildcat_forward_binned(
            qp, kp, vp, BH, m, n, d, float(beta), int(r), int(nbins), int(bool(recenter)),
            float(tau), int(seed), float(eps), sfp, rp, nr,
            O.ctypes.data_as(_f64p), S.ctypes.data_as(_i32p), rank.ctypes.data_as(_i32p))
        if err == 2:
            raise ValueError("n and r must be multiples of nbins")
        if err:
            raise MemoryError("oracle_wildcat_forward_binned")
        return O, S, rank


    def decode_attend(self, Qn, Kn, Vn, KS, VS, w, rank, vmin, vmax, beta):
        """New tokens over the compressed cache plus causal exact attention
        among themselves (Sec. 2, KV-cache decode).  Returns O [BH, m, d]."""
        Qn, qp = self._f64(Qn)
        Kn, kp = self._f64(Kn)
        Vn, vp = self._f64(Vn)
        KS, ksp = self._f64(KS)
        VS, vsp = self._f64(VS)
        w, wp = self._f64(w)
        rank, rkp = self._i32(rank)
        vmin, lop = self._f64(vmin)
        vmax, hip = self._f64(vmax)
        BH, m, d = Qn.shape
        r = KS.shape[1]
        O = np.zeros((BH, m, d))
        err = self.lib.oracle_decode_attend(qp, kp, vp, ksp, vsp, wp, rkp, lop, hip, BH, m, d, r,
                                            float(beta), O.ctypes.data_as(_f64p))
        if err:
            raise MemoryError("oracle_decode_attend")
        return O


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from the unmodified source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
