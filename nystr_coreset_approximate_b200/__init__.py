"""WildCat weighted-coreset attention on B200 (sm_100a): thin Python binding.

Every call marshals torch tensors into the C ABI of ``libwildcat.so``
(declared in ``include/wildcat.h``) and enqueues the library's CUDA kernels
on the current torch stream.  Nothing here computes any part of the method;
torch only provides device memory and streams.  There is no fallback: if
the library is missing, or a tensor is not on a CUDA device, the call
raises.

Method: "WildCat: Near-Linear Attention in Theory and Practice"
(Schroeder & Mackey), Sec. 2 and Alg. 1-4.

    S, F, rank, K_S = select(K, beta, r, seed)              # Alg. 1 RPNys
    V_S, w, vmin, vmax = weights(F, S, rank, V)             # Alg. 2 CompressKV
    O_hat = attend(Q, K_S, rank, beta, V_S, w, vmin, vmax)  # Alg. 3 WtdAttn
    O_hat, S, rank = forward(Q, K, V, beta, r, seed)        # Alg. 4 WildCat
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

__all__ = [
    "WildcatError", "library_path", "lib", "declared_symbols", "select", "select_fixed",
    "weights", "weights_inverse", "attend", "attend_noalloc", "decode_attend", "forward", "forward_ex", "Options", "forward_binned", "BinnedForwardPlan", "forward_host", "ForwardPlan", "pivot_uniforms",
    "set_select_cluster", "last_select_cluster", "set_select_kernel", "last_select_kernel",
    "force_select_timeout", "last_select_threads", "set_select_phase_steps", "last_select_phases",
    "set_stage_events",
    "device_status", "DTYPES",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_HEADER = os.path.join(os.path.dirname(_HERE), "include", "wildcat.h")

DTYPES = {"f32": 0, "bf16": 1}

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_f32 = ctypes.c_float
_u64 = ctypes.c_uint64
_sz = ctypes.c_size_t

_SIGS = {
    "wildcat_version": ([], _int),
    "wildcat_last_error": ([], ctypes.c_char_p),
    "wildcat_status_string": ([_int], ctypes.c_char_p),
    "wildcat_select": ([_vp, _int, _i64, _i64, _int, _f32, _int, _u64, _i64, _f32, _vp, _vp, _vp, _vp,
                        _vp], _int),
    "wildcat_select_fixed": ([_vp, _int, _i64, _i64, _int, _f32, _int, _f32, _vp, _vp, _vp, _vp, _vp,
                              _vp], _int),
    "wildcat_weights_workspace_size": ([_i64, _i64, _int, _int], _sz),
    "wildcat_weights": ([_vp, _vp, _vp, _vp, _int, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _sz,
                         _vp], _int),
    "wildcat_select_workspace_size": ([_i64, _i64], _sz),
    "wildcat_select_ws": ([_vp, _int, _i64, _i64, _int, _f32, _int, _u64, _i64, _f32, _vp, _vp, _vp, _vp, _vp,
                           _sz, _vp], _int),
    "wildcat_weights_inverse_workspace_size": ([_i64, _i64, _int, _int], _sz),
    "wildcat_weights_inverse": ([_vp, _vp, _int, _vp, _vp, _i64, _i64, _int, _int, _f32, _vp, _vp, _vp,
                                 _vp, _vp, _sz, _vp], _int),
    "wildcat_attend_workspace_size": ([_i64, _i64, _int, _int], _sz),
    "wildcat_attend": ([_vp, _vp, _int, _i64, _i64, _int, _int, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _vp,
                        _sz, _vp], _int),
    "wildcat_attend_noalloc": ([_vp, _vp, _int, _i64, _i64, _int, _int, _vp, _f32, _vp, _vp, _vp, _vp,
                                _vp, _vp], _int),
    "wildcat_decode_attend_workspace_size": ([_i64, _int], _sz),
    "wildcat_decode_attend": ([_vp, _vp, _vp, _vp, _int, _i64, _i64, _int, _int, _vp, _f32, _vp, _vp, _vp,
                               _vp, _vp, _vp, _sz, _vp], _int),
    "wildcat_forward_workspace_size": ([_i64, _i64, _i64, _int, _int, _int], _sz),
    "wildcat_forward": ([_vp, _vp, _vp, _int, _i64, _i64, _i64, _int, _f32, _int, _u64, _i64, _f32, _vp,
                         _vp, _vp, _vp, _sz, _vp], _int),
    "wildcat_forward_ex_workspace_size": ([_i64, _i64, _i64, _int, _int, _int, _vp], _sz),
    "wildcat_forward_ex": ([_vp, _vp, _vp, _int, _i64, _i64, _i64, _int, _f32, _int, _u64, _i64, _f32, _vp,
                            _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "wildcat_forward_binned_workspace_size": ([_i64, _i64, _i64, _int, _int, _int, _int], _sz),
    "wildcat_forward_binned": ([_vp, _vp, _vp, _int, _i64, _i64, _i64, _int, _f32, _int, _int, _u64, _i64,
                                _f32, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "wildcat_forward_host_workspace_size": ([_i64, _i64, _i64, _int, _int, _int], _sz),
    "wildcat_forward_host": ([_vp, _vp, _vp, _int, _i64, _i64, _i64, _int, _f32, _int, _u64, _i64, _f32,
                              _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "wildcat_forward_ex_host_workspace_size": ([_i64, _i64, _i64, _int, _int, _int, _vp], _sz),
    "wildcat_forward_ex_host": ([_vp, _vp, _vp, _int, _i64, _i64, _i64, _int, _f32, _int, _u64, _i64, _f32,
                                 _vp, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "wildcat_pivot_uniforms": ([_u64, _i64, _int, _vp, _vp], _int),
    "wildcat_get_device_status": ([_vp], _int),
    "wildcat_test_force_wait_timeout": ([_i64], _int),
    "wildcat_set_select_cluster": ([_int], _int),
    "wildcat_last_select_cluster": ([], _int),
    "wildcat_test_force_select_timeout": ([_i64], _int),
    "wildcat_set_select_kernel": ([_int], _int),
    "wildcat_last_select_kernel": ([], _int),
    "wildcat_last_select_threads": ([], _int),
    "wildcat_set_select_phase_steps": ([_int], _int),
    "wildcat_last_select_phases": ([], _int),
    "wildcat_set_stage_events": ([_vp, _vp], _int),
}


class WildcatError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libwildcat.so")


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libwildcat.so (built in-tree by ``build.py``); raise if absent."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"libwildcat.so not built ({path}); run "
                               "`python -m nystr_coreset_approximate_b200.build`")
        handle = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def declared_symbols():
    """Names of every function declared in include/wildcat.h."""
    with open(_HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wildcat_[a-z0-9_]+)\s*\(", text)))


def _check(status: int):
    if status != 0:
        raise WildcatError(status, lib().wildcat_last_error().decode())


# --------------------------------------------------------------------------- helpers
def _torch():
    import torch

    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return 0
    if t.dtype == torch.bfloat16:
        return 1
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dev(t, name, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    # the library launches on the current device (and keys per-device state on
    # it): a tensor elsewhere would be read through the wrong GPU
    cur = _torch().cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on cuda:{t.device.index} but the current device is cuda:{cur}; "
                         f"call under torch.cuda.device({t.device.index})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")
    return _vp(t.data_ptr())


def _opt(t, name, dtype=None):
    return None if t is None else _dev(t, name, dtype)


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return _vp(s.cuda_stream)


def _shape3(t, name):
    if t.dim() != 3:
        raise ValueError(f"{name} must be [BH, rows, d]")
    return t.shape


# --------------------------------------------------------------------------- calls
def select(K, beta: float, r: int, seed: int = 0, eps: float = 1e-6, *, inst0: int = 0, out=None,
           stream=None):
    """RPCholesky coreset selection (Alg. 1 RPNys).  K [BH, n, d] (float32 or
    bfloat16, CUDA).  inst0 is the global index of K's first instance (for a
    shard of a larger batch).  Returns (S [BH,r] int32, F [BH,r,n] float32,
    rank [BH] int32, K_S [BH,r,d])."""
    torch = _torch()
    BH, n, d = _shape3(K, "K")
    S, F, rank, K_S = out if out is not None else (
        torch.empty((BH, r), dtype=torch.int32, device=K.device),
        torch.empty((BH, r, n), dtype=torch.float32, device=K.device),
        torch.empty((BH,), dtype=torch.int32, device=K.device),
        torch.empty((BH, r, d), dtype=K.dtype, device=K.device))
    L = lib()
    nbytes = int(L.wildcat_select_workspace_size(BH, n))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=K.device)
    _check(L.wildcat_select_ws(_dev(K, "K"), _dtype_code(K), BH, n, d, float(beta), int(r),
                               int(seed) & (2**64 - 1), int(inst0), float(eps),
                               _dev(S, "S", torch.int32),
                               _dev(F, "F", torch.float32), _dev(rank, "rank", torch.int32),
                               _opt(K_S, "K_S", K.dtype), _dev(ws, "workspace"), nbytes, _stream(stream)))
    return S, F, rank, K_S


def select_fixed(K, beta: float, S_fixed, eps: float = 1e-6, *, stream=None):
    """The factorisation on given pivots S_fixed [BH, r] int32 (test entry point)."""
    torch = _torch()
    BH, n, d = _shape3(K, "K")
    r = S_fixed.shape[1]
    S = torch.empty((BH, r), dtype=torch.int32, device=K.device)
    F = torch.empty((BH, r, n), dtype=torch.float32, device=K.device)
    rank = torch.empty((BH,), dtype=torch.int32, device=K.device)
    K_S = torch.empty((BH, r, d), dtype=K.dtype, device=K.device)
    _check(lib().wildcat_select_fixed(_dev(K, "K"), _dtype_code(K), BH, n, d, float(beta), int(r),
                                      float(eps), _dev(S_fixed, "S_fixed", torch.int32),
                                      _dev(S, "S"), _dev(F, "F"), _dev(rank, "rank"),
                                      _dev(K_S, "K_S"), _stream(stream)))
    return S, F, rank, K_S


def weights(F, S, rank, V, *, stream=None):
    """Nystrom weights on (V, 1_n) (Alg. 2 CompressKV).  Returns (V_S [BH,r,d],
    w [BH,r], vmin [BH,d], vmax [BH,d]), all float32."""
    torch = _torch()
    BH, n, d = _shape3(V, "V")
    r = F.shape[1]
    dev = V.device
    V_S = torch.empty((BH, r, d), dtype=torch.float32, device=dev)
    w = torch.empty((BH, r), dtype=torch.float32, device=dev)
    vmin = torch.empty((BH, d), dtype=torch.float32, device=dev)
    vmax = torch.empty((BH, d), dtype=torch.float32, device=dev)
    L = lib()
    nbytes = int(L.wildcat_weights_workspace_size(BH, n, d, r))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(L.wildcat_weights(_dev(F, "F", torch.float32), _dev(S, "S", torch.int32),
                             _dev(rank, "rank", torch.int32), _dev(V, "V"), _dtype_code(V), BH, n, d,
                             r, _dev(V_S, "V_S"), _dev(w, "w"), _dev(vmin, "vmin"),
                             _dev(vmax, "vmax"), _dev(ws, "workspace"), nbytes, _stream(stream)))
    return V_S, w, vmin, vmax


def weights_inverse(K, S, rank, V, beta: float, *, stream=None):
    """The Nystrom weights through the maintained inverse of h(K_S, K_S) (Sec. 2,
    RPNys rank-one update), fp64 inside.  Same outputs as weights():
    (V_S [BH,r,d], w [BH,r], vmin [BH,d], vmax [BH,d]), float32."""
    torch = _torch()
    BH, n, d = _shape3(V, "V")
    r = S.shape[1]
    dev = V.device
    V_S = torch.empty((BH, r, d), dtype=torch.float32, device=dev)
    w = torch.empty((BH, r), dtype=torch.float32, device=dev)
    vmin = torch.empty((BH, d), dtype=torch.float32, device=dev)
    vmax = torch.empty((BH, d), dtype=torch.float32, device=dev)
    L = lib()
    nbytes = int(L.wildcat_weights_inverse_workspace_size(BH, n, d, r))
    if nbytes == 0:
        raise ValueError("weights_inverse supports 1 <= r <= 2048")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(L.wildcat_weights_inverse(_dev(K, "K"), _dev(V, "V"), _dtype_code(V), _dev(S, "S", torch.int32),
                                     _dev(rank, "rank", torch.int32), BH, n, d, r, float(beta),
                                     _dev(V_S, "V_S"), _dev(w, "w"), _dev(vmin, "vmin"), _dev(vmax, "vmax"),
                                     _dev(ws, "workspace"), nbytes, _stream(stream)))
    return V_S, w, vmin, vmax


def attend(Q, K_S, rank, beta: float, V_S, w, vmin, vmax, *, stream=None):
    """Weighted-coreset attention with value-range clip (Alg. 3 WtdAttn).
    Returns O_hat [BH, m, d] float32."""
    torch = _torch()
    BH, m, d = _shape3(Q, "Q")
    r = K_S.shape[1]
    if K_S.dtype != Q.dtype:
        raise TypeError("Q and K_S must share a dtype")
    O = torch.empty((BH, m, d), dtype=torch.float32, device=Q.device)
    L = lib()
    nbytes = int(L.wildcat_attend_workspace_size(BH, m, d, r))
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=Q.device)
    _check(L.wildcat_attend(_dev(Q, "Q"), _dev(K_S, "K_S"), _dtype_code(Q), BH, m, d, r,
                            _dev(rank, "rank", torch.int32), float(beta),
                            _dev(V_S, "V_S", torch.float32), _dev(w, "w", torch.float32),
                            _dev(vmin, "vmin", torch.float32), _dev(vmax, "vmax", torch.float32),
                            _dev(O, "O"), _dev(ws, "workspace"), nbytes, _stream(stream)))
    return O


def attend_noalloc(Q, K_S, rank, beta: float, V_S, w, vmin, vmax, *, out=None, stream=None):
    """wildcat_attend_noalloc: the same result as ``attend`` from a library
    call that allocates nothing (its scratch is a static 1 MiB device array;
    for callers that cannot allocate device memory).  ``out`` (optional) is
    the caller's O [BH, m, d] float32; without it torch allocates O here,
    outside the library call."""
    torch = _torch()
    BH, m, d = _shape3(Q, "Q")
    r = K_S.shape[1]
    if K_S.dtype != Q.dtype:
        raise TypeError("Q and K_S must share a dtype")
    O = out if out is not None else torch.empty((BH, m, d), dtype=torch.float32, device=Q.device)
    _check(lib().wildcat_attend_noalloc(_dev(Q, "Q"), _dev(K_S, "K_S"), _dtype_code(Q), BH, m, d, r,
                                        _dev(rank, "rank", torch.int32), float(beta),
                                        _dev(V_S, "V_S", torch.float32), _dev(w, "w", torch.float32),
                                        _dev(vmin, "vmin", torch.float32),
                                        _dev(vmax, "vmax", torch.float32),
                                        _dev(O, "O", torch.float32), _stream(stream)))
    return O


def decode_attend(Q_new, K_new, V_new, K_S, rank, beta: float, V_S, w, vmin, vmax, *, stream=None):
    """KV-cache decode with new tokens: Q_new/K_new/V_new [BH, m, d] attend
    over the compressed cache (K_S, V_S, w, rank, vmin, vmax) and causally
    over the new tokens.  Returns O [BH, m, d] float32."""
    torch = _torch()
    BH, m, d = _shape3(Q_new, "Q_new")
    r = K_S.shape[1]
    for t, nm in ((K_new, "K_new"), (V_new, "V_new"), (K_S, "K_S")):
        if t.dtype != Q_new.dtype:
            raise TypeError(f"{nm} must share Q_new's dtype")
    O = torch.empty((BH, m, d), dtype=torch.float32, device=Q_new.device)
    L = lib()
    nbytes = int(L.wildcat_decode_attend_workspace_size(BH, d))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=Q_new.device)
    _check(L.wildcat_decode_attend(_dev(Q_new, "Q_new"), _dev(K_new, "K_new"), _dev(V_new, "V_new"),
                                   _dev(K_S, "K_S"), _dtype_code(Q_new), BH, m, d, r,
                                   _dev(rank, "rank", torch.int32), float(beta),
                                   _dev(V_S, "V_S", torch.float32), _dev(w, "w", torch.float32),
                                   _dev(vmin, "vmin", torch.float32), _dev(vmax, "vmax", torch.float32),
                                   _dev(O, "O"), _dev(ws, "workspace"), nbytes, _stream(stream)))
    return O


class ForwardPlan:
    """Preallocated workspace and outputs for repeated wildcat_forward calls
    on one shape (what a serving loop or the benchmark holds on to)."""

    def __init__(self, BH, m, n, d, r, dtype: str, device="cuda"):
        torch = _torch()
        self.BH, self.m, self.n, self.d, self.r = BH, m, n, d, r
        self.code = DTYPES[dtype]
        L = lib()
        self.ws_bytes = int(L.wildcat_forward_workspace_size(BH, m, n, d, r, self.code))
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.O = torch.empty((BH, m, d), dtype=torch.float32, device=device)
        self.S = torch.empty((BH, r), dtype=torch.int32, device=device)
        self.rank = torch.empty((BH,), dtype=torch.int32, device=device)

    def run(self, Q, K, V, beta, seed, eps=1e-6, stream=None, inst0=0):
        _check(lib().wildcat_forward(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), self.code, self.BH,
                                     self.m, self.n, self.d, float(beta), self.r,
                                     int(seed) & (2**64 - 1), int(inst0), float(eps),
                                     _dev(self.O, "O"),
                                     _dev(self.S, "S"), _dev(self.rank, "rank"),
                                     _dev(self.ws, "workspace"), self.ws_bytes, _stream(stream)))
        return self.O, self.S, self.rank


def forward(Q, K, V, beta: float, r: int, seed: int = 0, eps: float = 1e-6, *, inst0: int = 0,
            stream=None):
    """The whole WildCat module (Alg. 4).  Returns (O_hat, S, rank).  inst0:
    global index of the first instance (for a shard of a larger batch)."""
    BH, m, d = _shape3(Q, "Q")
    n = K.shape[1]
    code = _dtype_code(K)
    if Q.dtype != K.dtype or V.dtype != K.dtype:
        raise TypeError("Q, K, V must share a dtype")
    plan = ForwardPlan(BH, m, n, d, r, "bf16" if code else "f32", device=K.device)
    O, S, rank = plan.run(Q, K, V, beta, seed, eps, stream, inst0)
    return O.clone(), S.clone(), rank.clone()


class BinnedForwardPlan:
    """Preallocated workspace and outputs for wildcat_forward_binned."""

    def __init__(self, BH, m, n, d, r, nbins, dtype: str, device="cuda"):
        torch = _torch()
        self.BH, self.m, self.n, self.d, self.r, self.nbins = BH, m, n, d, r, nbins
        self.code = DTYPES[dtype]
        L = lib()
        self.ws_bytes = int(L.wildcat_forward_binned_workspace_size(BH, m, n, d, r, nbins, self.code))
        if self.ws_bytes == 0:
            raise ValueError("n and r must be multiples of nbins")
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.O = torch.empty((BH, m, d), dtype=torch.float32, device=device)
        self.S = torch.empty((BH, r), dtype=torch.int32, device=device)
        self.rank = torch.empty((BH, nbins), dtype=torch.int32, device=device)

    def run(self, Q, K, V, beta, seed, eps=1e-6, stream=None, inst0=0):
        _check(lib().wildcat_forward_binned(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), self.code, self.BH,
                                            self.m, self.n, self.d, float(beta), self.r, self.nbins,
                                            int(seed) & (2**64 - 1), int(inst0), float(eps),
                                            _dev(self.O, "O"), _dev(self.S, "S"), _dev(self.rank, "rank"),
                                            _dev(self.ws, "workspace"), self.ws_bytes, _stream(stream)))
        return self.O, self.S, self.rank


def forward_binned(Q, K, V, beta: float, r: int, nbins: int, seed: int = 0, eps: float = 1e-6, *,
                   inst0: int = 0, stream=None):
    """WildCat with divide-and-conquer binning (Sec. 2): nbins contiguous key
    bins with r / nbins pivots each.  Returns (O_hat, S [BH, r] global key
    indices, rank [BH, nbins])."""
    BH, m, d = _shape3(Q, "Q")
    n = K.shape[1]
    code = _dtype_code(K)
    plan = BinnedForwardPlan(BH, m, n, d, r, nbins, "bf16" if code else "f32", device=K.device)
    O, S, rank = plan.run(Q, K, V, beta, seed, eps, stream, inst0)
    return O.clone(), S.clone(), rank.clone()


class Options(ctypes.Structure):
    """wildcat_options: divide-and-conquer bins, key recentring, temperature."""
    _fields_ = [("nbins", ctypes.c_int), ("recenter", ctypes.c_int), ("tau", ctypes.c_float)]


def forward_ex(Q, K, V, beta: float, r: int, seed: int = 0, eps: float = 1e-6, *, nbins: int = 1,
               recenter: bool = False, tau: float = 1.0, inst0: int = 0, stream=None):
    """WildCat with the options of Sec. 2 (bins, recentring, temperature).
    Returns (O_hat, S [BH, r] global key indices, rank [BH, nbins])."""
    torch = _torch()
    BH, m, d = _shape3(Q, "Q")
    n = K.shape[1]
    code = _dtype_code(K)
    opts = Options(int(nbins), int(bool(recenter)), float(tau))
    L = lib()
    nbytes = int(L.wildcat_forward_ex_workspace_size(BH, m, n, d, r, code, ctypes.byref(opts)))
    if nbytes == 0:
        raise ValueError("n and r must be multiples of nbins")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=K.device)
    O = torch.empty((BH, m, d), dtype=torch.float32, device=K.device)
    S = torch.empty((BH, r), dtype=torch.int32, device=K.device)
    rank = torch.empty((BH, nbins), dtype=torch.int32, device=K.device)
    _check(L.wildcat_forward_ex(_dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), code, BH, m, n, d, float(beta), int(r),
                                int(seed) & (2**64 - 1), int(inst0), float(eps), ctypes.byref(opts),
                                _dev(O, "O"), _dev(S, "S"), _dev(rank, "rank"), _dev(ws, "workspace"), nbytes,
                                _stream(stream)))
    return O, S, rank


class HostForwardPlan:
    """Device workspace for wildcat_forward_host (inputs and outputs in host memory)."""

    def __init__(self, BH, m, n, d, r, dtype: str, device="cuda"):
        torch = _torch()
        self.BH, self.m, self.n, self.d, self.r = BH, m, n, d, r
        self.code = DTYPES[dtype]
        L = lib()
        self.ws_bytes = int(L.wildcat_forward_host_workspace_size(BH, m, n, d, r, self.code))
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)

    def run(self, Q_host, K_host, V_host, O_host, beta, seed, eps=1e-6, S_host=None,
            rank_host=None, stream=None, inst0=0):
        for t, nm in ((Q_host, "Q"), (K_host, "K"), (V_host, "V"), (O_host, "O")):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{nm} must be a contiguous host tensor")
        _check(lib().wildcat_forward_host(
            _vp(Q_host.data_ptr()), _vp(K_host.data_ptr()), _vp(V_host.data_ptr()), self.code,
            self.BH, self.m, self.n, self.d, float(beta), self.r, int(seed) & (2**64 - 1),
            int(inst0), float(eps), _vp(O_host.data_ptr()),
            None if S_host is None else _vp(S_host.data_ptr()),
            None if rank_host is None else _vp(rank_host.data_ptr()),
            _dev(self.ws, "workspace"), self.ws_bytes, _stream(stream)))
        return O_host


def forward_host(Q_host, K_host, V_host, beta: float, r: int, seed: int = 0, eps: float = 1e-6):
    """wildcat_forward on host tensors (copies in, computes on the GPU, copies out)."""
    torch = _torch()
    BH, m, d = _shape3(Q_host, "Q")
    n = K_host.shape[1]
    plan = HostForwardPlan(BH, m, n, d, r, "bf16" if _dtype_code(K_host) else "f32")
    O = torch.empty((BH, m, d), dtype=torch.float32).pin_memory()
    S = torch.empty((BH, r), dtype=torch.int32)
    rank = torch.empty((BH,), dtype=torch.int32)
    plan.run(Q_host, K_host, V_host, O, beta, seed, eps, S, rank)
    return O, S, rank


class HostForwardExPlan:
    """Device workspace for wildcat_forward_ex_host (the forward with the
    options of Sec. 2; inputs and outputs in host memory)."""

    def __init__(self, BH, m, n, d, r, dtype: str, nbins: int = 1, recenter: bool = False, tau: float = 1.0,
                 device="cuda"):
        torch = _torch()
        self.BH, self.m, self.n, self.d, self.r = BH, m, n, d, r
        self.code = DTYPES[dtype]
        self.opts = Options(int(nbins), int(bool(recenter)), float(tau))
        L = lib()
        self.ws_bytes = int(L.wildcat_forward_ex_host_workspace_size(BH, m, n, d, r, self.code,
                                                                      ctypes.byref(self.opts)))
        if self.ws_bytes == 0:
            raise ValueError("n and r must be multiples of nbins")
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)

    def run(self, Q_host, K_host, V_host, O_host, beta, seed, eps=1e-6, S_host=None,
            rank_host=None, stream=None, inst0=0):
        for t, nm in ((Q_host, "Q"), (K_host, "K"), (V_host, "V"), (O_host, "O")):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{nm} must be a contiguous host tensor")
        _check(lib().wildcat_forward_ex_host(
            _vp(Q_host.data_ptr()), _vp(K_host.data_ptr()), _vp(V_host.data_ptr()), self.code,
            self.BH, self.m, self.n, self.d, float(beta), self.r, int(seed) & (2**64 - 1),
            int(inst0), float(eps), ctypes.byref(self.opts), _vp(O_host.data_ptr()),
            None if S_host is None else _vp(S_host.data_ptr()),
            None if rank_host is None else _vp(rank_host.data_ptr()),
            _dev(self.ws, "workspace"), self.ws_bytes, _stream(stream)))
        return O_host


def forward_ex_host(Q_host, K_host, V_host, beta: float, r: int, seed: int = 0, eps: float = 1e-6, *,
                    nbins: int = 1, recenter: bool = False, tau: float = 1.0):
    """wildcat_forward_ex on host tensors.  Returns (O_hat, S [BH, r], rank [BH, nbins]) on the host."""
    torch = _torch()
    BH, m, d = _shape3(Q_host, "Q")
    n = K_host.shape[1]
    plan = HostForwardExPlan(BH, m, n, d, r, "bf16" if _dtype_code(K_host) else "f32", nbins, recenter, tau)
    O = torch.empty((BH, m, d), dtype=torch.float32).pin_memory()
    S = torch.empty((BH, r), dtype=torch.int32)
    rank = torch.empty((BH, nbins), dtype=torch.int32)
    plan.run(Q_host, K_host, V_host, O, beta, seed, eps, S, rank)
    return O, S, rank


def pivot_uniforms(seed: int, BH: int, steps: int, device="cuda"):
    """The pivot uniforms u[b, i] the select kernels draw (float64, device)."""
    torch = _torch()
    u = torch.empty((BH, steps), dtype=torch.float64, device=device)
    _check(lib().wildcat_pivot_uniforms(int(seed) & (2**64 - 1), BH, steps, _dev(u, "u"),
                                        _stream()))
    return u


def device_status(stream=None) -> int:
    """Wait for the stream, then return and clear the device status word
    (0 = fine, 5 = a kernel's bounded wait expired)."""
    return int(lib().wildcat_get_device_status(_stream(stream)))


def set_select_cluster(G: int):
    """CTAs per instance in the select kernel (0 = automatic)."""
    _check(lib().wildcat_set_select_cluster(int(G)))


def last_select_cluster() -> int:
    return int(lib().wildcat_last_select_cluster())


def set_select_kernel(kernel: int):
    """0 = automatic, 1 = the select kernel on clusters, 3 = its global-sync
    form where it applies."""
    _check(lib().wildcat_set_select_kernel(int(kernel)))


def last_select_kernel() -> int:
    """1 = clusters, 3 = global sync (form of the last select launch)."""
    return int(lib().wildcat_last_select_kernel())


def last_select_threads() -> int:
    """Threads per CTA of the last select launch (256 or 512)."""
    return int(lib().wildcat_last_select_threads())


def set_select_phase_steps(steps: int):
    """Steps per select launch when a workspace is given: 0 = automatic
    (64 for r >= 512), > 0 = that many, < 0 = one launch."""
    _check(lib().wildcat_set_select_phase_steps(int(steps)))


def last_select_phases() -> int:
    """Launches of the last select call (1 = no phases)."""
    return int(lib().wildcat_last_select_phases())


def set_stage_events(after_select=None, after_weights=None):
    """Stage markers for the forward calls on this thread: torch.cuda.Event
    objects (each recorded once already, so that its handle exists) that a
    forward records right after its select and right after its weights;
    None turns a marker off."""
    def handle(ev):
        if ev is None:
            return None
        h = int(ev.cuda_event)
        if h == 0:
            raise ValueError("record the event once before passing it (its handle is created lazily)")
        return h
    _check(lib().wildcat_set_stage_events(handle(after_select), handle(after_weights)))


def force_select_timeout(nanoseconds: int):
    """Test hook: the select's global-sync barrier waits this long on a
    counter one CTA never bumps (0 = off)."""
    _check(lib().wildcat_test_force_select_timeout(int(nanoseconds)))
