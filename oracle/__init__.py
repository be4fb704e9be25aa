"""Oracle for SATA attention: plain float64 C (``sata_oracle.c``) behind ctypes.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the library and its
Python binding never do.  It shares no code with the CUDA path.

Every routine is pinned by the CPU tests against something other than itself
(closed forms, brute force over the full tensor power, exact integer identities,
special cases, the softmax limit); see ``tests/test_oracle_pins.py``.

Page references (by title and section):
  [CC-TAYLOR] "Self-attention at constant cost per token via symmetry-aware
              Taylor approximation" (blog.hotdry.top, 2026-02-05)
  [CC-HW]     "Constant-cost attention: hardware optimization" (same blog)
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sata_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_llp = ctypes.POINTER(ctypes.c_longlong)


def build(force: bool = False) -> str:
    """Compile the oracle's C source into ``oracle/liboracle.so`` (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_binom.restype = ctypes.c_longlong
            lib.oracle_binom.argtypes = [ctypes.c_int, ctypes.c_int]
            lib.oracle_num_features.restype = ctypes.c_longlong
            lib.oracle_num_features.argtypes = [ctypes.c_int, ctypes.c_int]
            lib.oracle_basis.restype = ctypes.c_longlong
            lib.oracle_basis.argtypes = [ctypes.c_int, ctypes.c_int, _ip, _ip, _llp, _llp]
            lib.oracle_features.restype = ctypes.c_int
            lib.oracle_features.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _dp]
            lib.oracle_scan.restype = ctypes.c_int
            lib.oracle_scan.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                        ctypes.c_longlong, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.oracle_direct.restype = ctypes.c_int
            lib.oracle_direct.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_longlong, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.oracle_direct_at.restype = ctypes.c_int
            lib.oracle_direct_at.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                             ctypes.c_longlong, _dp, _dp, _dp, ctypes.c_longlong, ctypes.c_void_p,
                                             _dp, _dp, _dp]
            lib.oracle_direct_grad.restype = ctypes.c_int
            lib.oracle_direct_grad.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                               ctypes.c_longlong, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.oracle_softmax.restype = ctypes.c_int
            lib.oracle_softmax.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_longlong, _dp, _dp, _dp, _dp]
            lib.oracle_costs.restype = ctypes.c_int
            lib.oracle_costs.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _llp, _llp]
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: widen exactly (bf16/fp32 -> fp64)
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    if a.dtype == np.float64:
        return a.ctypes.data_as(_dp)
    if a.dtype == np.int32:
        return a.ctypes.data_as(_ip)
    if a.dtype == np.int64:
        return a.ctypes.data_as(_llp)
    raise TypeError(a.dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def default_c(d_K: int) -> float:
    """c = sqrt(d_K) ([CC-TAYLOR] "The Taylor approximation")."""
    return math.sqrt(d_K)


def num_features(d: int, P: int) -> int:
    return int(_load().oracle_num_features(d, P))


def basis(d: int, P: int):
    """Minimal basis: (deg [F] int32, M [F, max(P-1,1)] int32 padded with -1,
    C [F] int64, offsets [P+1] int64).  Lexicographic nondecreasing tuples,
    degrees concatenated p = 0..P-1."""
    lib = _load()
    F = int(lib.oracle_num_features(d, P))
    width = max(P - 1, 1)
    deg = np.zeros(F, np.int32)
    M = np.zeros((F, width), np.int32)
    C = np.zeros(F, np.int64)
    off = np.zeros(P + 1, np.int64)
    got = lib.oracle_basis(d, P, _ptr(deg), _ptr(M), _ptr(C), _ptr(off))
    if got != F:
        raise RuntimeError(f"oracle_basis returned {got}, expected {F}")
    return deg, M, C, off


def features(d: int, P: int, x) -> np.ndarray:
    """phi(x) over the whole truncated basis (unweighted)."""
    x = _f64(x)
    assert x.shape == (d,)
    out = np.zeros(num_features(d, P), np.float64)
    _check(_load().oracle_features(d, P, _ptr(x), _ptr(out)), "features")
    return out


def scan(q, k, v, P: int, c: float | None = None, S=None, Z=None):
    """The recurrence for one head over T tokens, continuing from (S, Z).

    q, k: [T, d_K]; v: [T, d_V].  Returns (y [T, d_V], den [T], S [F, d_V], Z [F]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, dK = q.shape
    dV = v.shape[1]
    c = default_c(dK) if c is None else float(c)
    F = num_features(dK, P)
    S = np.zeros((F, dV)) if S is None else _f64(S).copy()
    Z = np.zeros(F) if Z is None else _f64(Z).copy()
    y = np.zeros((T, dV))
    den = np.zeros(T)
    _check(_load().oracle_scan(dK, dV, P, c, T, _ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(Z),
                               _ptr(y), _ptr(den)), "scan")
    return y, den, S, Z


def direct(q, k, v, P: int, c: float | None = None):
    """Masked O(T^2) truncated-Taylor attention for one head: (y, den, kappa)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, dK = q.shape
    dV = v.shape[1]
    c = default_c(dK) if c is None else float(c)
    y = np.zeros((T, dV))
    den = np.zeros(T)
    kappa = np.zeros(T)
    _check(_load().oracle_direct(dK, dV, P, c, T, _ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(den),
                                 _ptr(kappa)), "direct")
    return y, den, kappa


def direct_at(q, k, v, P: int, ts, c: float | None = None):
    """``direct`` at the token indices ``ts`` only, for one head: (y [n, d_V], den, kappa).

    Each output costs O(t d), so tokens deep into a long sequence can be checked."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, dK = q.shape
    dV = v.shape[1]
    c = default_c(dK) if c is None else float(c)
    idx = np.ascontiguousarray(np.asarray(ts, dtype=np.int64))
    n = idx.shape[0]
    y = np.zeros((n, dV))
    den = np.zeros(n)
    kappa = np.zeros(n)
    _check(_load().oracle_direct_at(dK, dV, P, c, T, _ptr(q), _ptr(k), _ptr(v), n,
                                    idx.ctypes.data_as(ctypes.c_void_p), _ptr(y), _ptr(den), _ptr(kappa)),
           "direct_at")
    return y, den, kappa


def direct_grad(q, k, v, dy, P: int, c: float | None = None):
    """Gradient of sum(dy * y) for the direct form of one head: (dq, dk, dv).

    q, k: [T, d_K]; v, dy: [T, d_V].  The exact chain rule through y = num/den
    (the pages define no backward pass; see ``oracle_direct_grad``)."""
    q, k, v, dy = _f64(q), _f64(k), _f64(v), _f64(dy)
    T, dK = q.shape
    dV = v.shape[1]
    c = default_c(dK) if c is None else float(c)
    dq = np.zeros((T, dK))
    dk = np.zeros((T, dK))
    dv = np.zeros((T, dV))
    _check(_load().oracle_direct_grad(dK, dV, P, c, T, _ptr(q), _ptr(k), _ptr(v), _ptr(dy),
                                      _ptr(dq), _ptr(dk), _ptr(dv)), "direct_grad")
    return dq, dk, dv


def grad_heads(q, k, v, dy, P: int, heads=None, T: int | None = None, threads: int | None = None,
               c: float | None = None):
    """``direct_grad`` for several heads of [B, H, N, d] inputs in parallel threads.

    Returns {(b, h): (dq, dk, dv)} over the first T tokens of each head."""
    q, k, v, dy = _f64(q), _f64(k), _f64(v), _f64(dy)
    B, H, N, _ = q.shape
    T = N if T is None else int(T)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    threads = threads or len(os.sched_getaffinity(0))

    def one(bh):
        b, h = bh
        return bh, direct_grad(q[b, h, :T], k[b, h, :T], v[b, h, :T], dy[b, h, :T], P, c)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        return dict(ex.map(one, heads))


def softmax(q, k, v, c: float | None = None) -> np.ndarray:
    """Exact causal softmax attention for one head (the P -> infinity limit)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, dK = q.shape
    dV = v.shape[1]
    c = default_c(dK) if c is None else float(c)
    y = np.zeros((T, dV))
    _check(_load().oracle_softmax(dK, dV, c, T, _ptr(q), _ptr(k), _ptr(v), _ptr(y)), "softmax")
    return y


def costs(dK: int, dV: int, P: int):
    """(state values, FLOPs per token) for one head, summed term by term."""
    st = ctypes.c_longlong(0)
    fl = ctypes.c_longlong(0)
    _check(_load().oracle_costs(dK, dV, P, ctypes.byref(st), ctypes.byref(fl)), "costs")
    return int(st.value), int(fl.value)


def prefill(q, k, v, P: int, heads=None, T: int | None = None, threads: int | None = None,
            c: float | None = None):
    """Run ``scan`` for several heads of [B, H, N, d] inputs in parallel threads
    (ctypes drops the GIL during each C call).

    heads: list of (b, h) pairs (default: all); T: tokens per head from the start
    (default: all).  Returns {(b, h): (y, den, S, Z)}.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, _ = q.shape
    T = N if T is None else int(T)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    threads = threads or len(os.sched_getaffinity(0))

    def one(bh):
        b, h = bh
        return bh, scan(q[b, h, :T], k[b, h, :T], v[b, h, :T], P, c)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        return dict(ex.map(one, heads))
