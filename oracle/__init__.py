"""Float64 CPU oracle for the DashAttention forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  The product path (the CUDA library and its binding)
never does.  The arithmetic lives in ``dash_oracle.c`` (plain C, double precision); this module
only builds it, loads it and marshals numpy arrays.

Formulas follow "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention"
(xllm-io paper review page, section 3): the alpha-entmax background formula, Eq. 4 (Stage 0),
Eq. 6 (Stage 1 with the GQA average), Eq. 9 / Eq. 11-12 and Proposition 4.1 (Stage 2).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dash_oracle.c")
_LIB = os.path.join(_HERE, "libdash_oracle.so")
_lib = None


class _Cfg(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("h_q", ctypes.c_int),
                ("h_kv", ctypes.c_int), ("d", ctypes.c_int), ("chunk", ctypes.c_int),
                ("alpha", ctypes.c_double), ("gamma", ctypes.c_double),
                ("inv_sigma", ctypes.c_double)]


def build(force: bool = False) -> str:
    """Compile dash_oracle.c into libdash_oracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        ip = ctypes.POINTER(ctypes.c_int)
        llp = ctypes.POINTER(ctypes.c_longlong)
        cfgp = ctypes.POINTER(_Cfg)
        lib.orc_entmax_threshold.argtypes = [dp, ctypes.c_int, ctypes.c_double]
        lib.orc_entmax_threshold.restype = ctypes.c_double
        lib.orc_entmax.argtypes = [dp, ctypes.c_int, ctypes.c_double, dp]
        lib.orc_entmax.restype = ctypes.c_int
        lib.orc_chunk_summary.argtypes = [cfgp, fp, llp, fp, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, dp]
        lib.orc_stage0.argtypes = [cfgp, fp, llp, fp, dp, ctypes.c_int]
        lib.orc_route_row.argtypes = [cfgp, fp, ctypes.c_longlong, dp, ctypes.c_int, dp, dp, dp]
        lib.orc_route_row.restype = ctypes.c_int
        lib.orc_rows.argtypes = [cfgp, fp, ip, ctypes.c_int, fp, llp, fp, llp, dp, ctypes.c_int,
                                 ctypes.c_int, dp, ip, dp, dp, dp, ctypes.c_int]
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_backward.argtypes = [cfgp, fp, fp, fp, fp, fp, dp, dp, dp, dp, ctypes.c_int]
        _lib = lib
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return _load().orc_num_threads()


def entmax(s, alpha: float) -> np.ndarray:
    """alpha-entmax of a 1-D score vector (background formula of the paper review page)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    p = np.zeros_like(s)
    _load().orc_entmax(_p(s, ctypes.c_double), s.size, float(alpha), _p(p, ctypes.c_double))
    return p


def entmax_threshold(x, alpha: float) -> float:
    """tau for x = (alpha-1)*s."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    return _load().orc_entmax_threshold(_p(x, ctypes.c_double), x.size, float(alpha))


def _cfg(batch, seqlen, h_q, h_kv, d, chunk, alpha, gamma, inv_sigma):
    return _Cfg(batch, seqlen, h_q, h_kv, d, chunk, float(alpha), float(gamma), float(inv_sigma))


def _strides(a):
    """Element strides [batch, position, head] of a [b, n, h, d] array with d contiguous."""
    assert a.ndim == 4 and a.strides[3] == a.itemsize
    return np.array([a.strides[0] // a.itemsize, a.strides[1] // a.itemsize,
                     a.strides[2] // a.itemsize], dtype=np.int64)


def stage0(K, qbar, chunk: int, nthreads: int = 0) -> np.ndarray:
    """Eq. 4 summaries of every complete chunk: returns kbar [b, h_kv, n//chunk, d] (float64)."""
    K = _f32(K)
    qbar = _f32(qbar)
    b, n, hkv, d = K.shape
    T = n // chunk
    kbar = np.zeros((b, hkv, T, d), dtype=np.float64)
    cf = _cfg(b, n, hkv, hkv, d, chunk, 1.5, 1.0, 1.0)
    ks = _strides(K)
    if T > 0:
        _load().orc_stage0(ctypes.byref(cf), _p(K, ctypes.c_float), _p(ks, ctypes.c_longlong),
                           _p(qbar, ctypes.c_float), _p(kbar, ctypes.c_double), int(nthreads))
    return kbar


def chunk_summary(K, qbar, b: int, r: int, t0: int, t1: int) -> np.ndarray:
    """Eq. 4 over keys t0..t1-1 (a running summary when the chunk is not complete yet)."""
    K = _f32(K)
    qbar = _f32(qbar)
    _, n, hkv, d = K.shape
    out = np.zeros(d, dtype=np.float64)
    cf = _cfg(K.shape[0], n, hkv, hkv, d, max(1, t1 - t0), 1.5, 1.0, 1.0)
    ks = _strides(K)
    _load().orc_chunk_summary(ctypes.byref(cf), _p(K, ctypes.c_float), _p(ks, ctypes.c_longlong),
                              _p(qbar, ctypes.c_float), b, r, t0, t1, _p(out, ctypes.c_double))
    return out


def route_counts(Qrows, pos, K, kbar, *, chunk, alpha, gamma, nthreads: int = 0):
    """Stage 1 only: |R| per (b, h_kv, row) for the given query rows (no Stage 2)."""
    Qrows = _f32(Qrows)
    b, nrows, hq, d = Qrows.shape
    hkv = kbar.shape[1]
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    T = kbar.shape[2]
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.int32), (b, nrows)))
    counts = np.zeros((b, hkv, nrows), dtype=np.int32)
    cf = _cfg(b, K.shape[1], hq, hkv, d, chunk, alpha, gamma, 1.0)
    dummy = np.zeros((1, 1, hkv, d), np.float32)
    st = _strides(dummy)
    nd = ctypes.POINTER(ctypes.c_double)()
    _load().orc_rows(ctypes.byref(cf), _p(Qrows, ctypes.c_float), _p(pos, ctypes.c_int), nrows,
                     _p(dummy, ctypes.c_float), _p(st, ctypes.c_longlong), _p(dummy, ctypes.c_float),
                     _p(st, ctypes.c_longlong), _p(kbar, ctypes.c_double), T, 0, nd,
                     _p(counts, ctypes.c_int), nd, nd, nd, int(nthreads))
    return counts


def rows(Qrows, pos, K, V, kbar, *, chunk, alpha, gamma, inv_sigma=1.0, prior_form=False,
         want_route=False, nthreads: int = 0):
    """Full forward for selected query rows.

    Qrows [b, nrows, h_q, d] are the query vectors, pos [b, nrows] their positions (int).
    K, V [b, n, h_kv, d]; kbar [b, h_kv, T, d] the Stage-0 summaries (T complete chunks).
    Returns O [b, nrows, h_q, d] float64, and with ``want_route`` also a dict with
    counts [b, h_kv, nrows] (|R|), w / bias / margin [b, h_kv, nrows, T] (0 past the visible
    chunks; margin = max over the group's heads of (alpha-1)*gamma*zbar - tau).
    """
    Qrows = _f32(Qrows)
    K = _f32(K) if K.dtype != np.float32 else K
    V = _f32(V) if V.dtype != np.float32 else V
    b, nrows, hq, d = Qrows.shape
    hkv = K.shape[2]
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    T = kbar.shape[2]
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.int32), (b, nrows)))
    O = np.zeros((b, nrows, hq, d), dtype=np.float64)
    cf = _cfg(b, K.shape[1], hq, hkv, d, chunk, alpha, gamma, inv_sigma)
    ks, vs = _strides(K), _strides(V)
    null_d = ctypes.POINTER(ctypes.c_double)()
    null_i = ctypes.POINTER(ctypes.c_int)()
    if want_route:
        counts = np.zeros((b, hkv, nrows), dtype=np.int32)
        w = np.zeros((b, hkv, nrows, T), dtype=np.float64)
        bias = np.zeros_like(w)
        margin = np.zeros_like(w)
        cp, wp, bp, mp = (_p(counts, ctypes.c_int), _p(w, ctypes.c_double),
                          _p(bias, ctypes.c_double), _p(margin, ctypes.c_double))
    else:
        cp, wp, bp, mp = null_i, null_d, null_d, null_d
    kbp = _p(kbar, ctypes.c_double) if kbar.size else ctypes.POINTER(ctypes.c_double)(ctypes.c_double(0.0))
    _load().orc_rows(ctypes.byref(cf), _p(Qrows, ctypes.c_float), _p(pos, ctypes.c_int), nrows,
                     _p(K, ctypes.c_float), _p(ks, ctypes.c_longlong), _p(V, ctypes.c_float),
                     _p(vs, ctypes.c_longlong), kbp, T, int(bool(prior_form)),
                     _p(O, ctypes.c_double), cp, wp, bp, mp, int(nthreads))
    if want_route:
        return O, {"counts": counts, "w": w, "bias": bias, "margin": margin}
    return O


def prefill(Q, K, V, qbar, *, chunk, alpha, gamma, inv_sigma=1.0, positions=None,
            prior_form=False, want_route=False, nthreads: int = 0):
    """Causal prefill forward over Q [b, n, h_q, d]; ``positions`` selects a subset of rows
    (all rows by default).  Returns (O rows, kbar[, route])."""
    b, n = Q.shape[0], Q.shape[1]
    kbar = stage0(K, qbar, chunk, nthreads)
    if positions is None:
        positions = np.arange(n, dtype=np.int32)
    positions = np.asarray(positions, dtype=np.int32)
    Qrows = Q[:, positions]
    res = rows(Qrows, np.broadcast_to(positions, (b, positions.size)), K, V, kbar, chunk=chunk,
               alpha=alpha, gamma=gamma, inv_sigma=inv_sigma, prior_form=prior_form,
               want_route=want_route, nthreads=nthreads)
    if want_route:
        return res[0], kbar, res[1]
    return res, kbar


def decode(q, K_cache, V_cache, qbar, seqlens, *, chunk, alpha, gamma, inv_sigma=1.0,
           want_route=False, nthreads: int = 0):
    """One decode step: the query q [b, h_q, d] sits at position seqlens[b]-1 of its sequence and
    sees cache positions 0..seqlens[b]-1 (its own key included).  Summaries are those of the
    complete chunks of the cache (Eq. 4).  Returns o [b, h_q, d] (float64)[, route]."""
    seqlens = np.asarray(seqlens, dtype=np.int64)
    b = q.shape[0]
    Lmax = int(seqlens.max())
    kbar = stage0(K_cache[:, :Lmax], qbar, chunk, nthreads)
    pos = (seqlens - 1).astype(np.int32).reshape(b, 1)
    res = rows(np.asarray(q)[:, None], pos, K_cache, V_cache, kbar, chunk=chunk, alpha=alpha,
               gamma=gamma, inv_sigma=inv_sigma, want_route=want_route, nthreads=nthreads)
    if want_route:
        return res[0][:, 0], res[1]
    return res[:, 0]


def backward(Q, K, V, qbar, dO, *, chunk, alpha, gamma, inv_sigma=1.0, nthreads: int = 0):
    """Gradients of L = sum(dO * O) for the causal prefill forward (prefill()) with respect to
    Q, K, V and qbar, in float64.  Q, dO [b, n, h_q, d]; K, V [b, n, h_kv, d]; qbar [h_kv, d].
    Returns dQ, dK, dV (same shapes) and dqbar [h_kv, d] (summed over the batch).  The routed
    support is held fixed (it is piecewise constant in the inputs)."""
    Q, K, V, qbar, dO = (_f32(a) for a in (Q, K, V, qbar, dO))
    b, n, hq, d = Q.shape
    hkv = K.shape[2]
    dQ = np.zeros(Q.shape, dtype=np.float64)
    dK = np.zeros(K.shape, dtype=np.float64)
    dV = np.zeros(V.shape, dtype=np.float64)
    dqbar = np.zeros((hkv, d), dtype=np.float64)
    cf = _cfg(b, n, hq, hkv, d, chunk, alpha, gamma, inv_sigma)
    _load().orc_backward(ctypes.byref(cf), _p(Q, ctypes.c_float), _p(K, ctypes.c_float), _p(V, ctypes.c_float),
                         _p(qbar, ctypes.c_float), _p(dO, ctypes.c_float), _p(dQ, ctypes.c_double),
                         _p(dK, ctypes.c_double), _p(dV, ctypes.c_double), _p(dqbar, ctypes.c_double),
                         int(nthreads))
    return dQ, dK, dV, dqbar
