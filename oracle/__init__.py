"""Plain float64 CPU oracle for alpha-entmax attention (ctypes binding).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library and its Python binding never import it, and the two
share no code.

The arithmetic lives in ``entmax_oracle.c`` (plain C, float64, OpenMP over
independent rows or heads).  Every function there cites the passage of the
AdaSplash pages it follows; this module only marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "entmax_oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP) if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        c_int, c_double = ctypes.c_int, ctypes.c_double
        lib.orc_entmax_tau.argtypes = [_dp, c_int, c_double, _dp]
        lib.orc_entmax_probs.argtypes = [_dp, c_int, c_double, c_double, _dp]
        lib.orc_entmax_row.argtypes = [_dp, c_int, c_double, _dp, _dp]
        lib.orc_sparsemax_tau_sort.argtypes = [_dp, c_int]
        lib.orc_sparsemax_tau_sort.restype = c_double
        lib.orc_entmax15_tau_sort.argtypes = [_dp, c_int]
        lib.orc_entmax15_tau_sort.restype = c_double
        lib.orc_entmax_vjp_row.argtypes = [_dp, c_int, c_double, c_double, _dp, _dp, _dp]
        lib.orc_entmax_vjp_row.restype = c_double
        lib.orc_attn_fwd.argtypes = [_dp, _dp, _dp, c_int, c_int, c_int, c_int, c_double,
                                     c_int, c_int, _dp, _dp, _dp, c_int]
        lib.orc_attn_fwd_rows.argtypes = [_dp, _dp, _dp, c_int, c_int, c_int, c_int, c_double,
                                          c_int, c_int, _i64p, c_int, _dp, _dp, _dp, c_int]
        lib.orc_attn_otilde_rows.argtypes = [_dp, _dp, _dp, c_int, c_int, c_int, c_int,
                                             c_double, c_int, _i64p, c_int, _dp, c_int]
        lib.orc_attn_bwd.argtypes = [_dp, _dp, _dp, _dp, c_int, c_int, c_int, c_int, c_double,
                                     c_int, _dp, _dp, _dp, _dp, _dp, c_int]
        lib.orc_attn_bwd_head_sampled.argtypes = [_dp, _dp, _dp, _dp, c_int, c_int, c_double,
                                                  c_int, _ip, c_int, _ip, c_int, _dp, _dp, _dp,
                                                  c_int]
        lib.orc_entmax_tau_iterative.argtypes = [_dp, c_int, c_double, c_int, c_int, c_double,
                                                 c_double, c_int, _dp, _ip]
        _lib = lib
    return _lib


def _d(a):
    """Contiguous float64 copy (or view) of ``a``."""
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a, t=_dp):
    return a.ctypes.data_as(t) if a is not None else None


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"oracle {name} rejected its arguments (rc={rc})")


# ---------------------------------------------------------------- row level
def entmax_tau(s, alpha):
    """tau of one score row (bisection to width 1e-12), in units of (alpha-1)*s."""
    s = _d(s)
    out = ctypes.c_double()
    _check(_L().orc_entmax_tau(_ptr(s), s.size, alpha, ctypes.byref(out)), "entmax_tau")
    return out.value


def entmax_probs(s, alpha, tau):
    s = _d(s)
    p = np.empty_like(s)
    _L().orc_entmax_probs(_ptr(s), s.size, alpha, tau, _ptr(p))
    return p


def entmax_row(s, alpha):
    """(p, tau) of one score row."""
    s = _d(s)
    p = np.empty_like(s)
    tau = ctypes.c_double()
    _check(_L().orc_entmax_row(_ptr(s), s.size, alpha, _ptr(p), ctypes.byref(tau)), "entmax_row")
    return p, tau.value


def sparsemax_tau_sort(s):
    s = _d(s)
    return _L().orc_sparsemax_tau_sort(_ptr(s), s.size)


def entmax15_tau_sort(s):
    s = _d(s)
    return _L().orc_entmax15_tau_sort(_ptr(s), s.size)


def entmax_vjp_row(s, alpha, tau, dp):
    """(ds, g, delta) of one row: ds = g*(dp - delta), delta = sum g dp / sum g."""
    s, dp = _d(s), _d(dp)
    ds, g = np.empty_like(s), np.empty_like(s)
    delta = _L().orc_entmax_vjp_row(_ptr(s), s.size, alpha, tau, _ptr(dp), _ptr(ds), _ptr(g))
    return ds, g, delta


def entmax_tau_iterative(s, alpha, method, nbins=64, ftol=1e-6, wtol=0.0, maxpass=64):
    """(tau, passes) by bisection (0), Halley-bisection (1) or histogram start (2)."""
    s = _d(s)
    tau = ctypes.c_double()
    passes = ctypes.c_int()
    _check(_L().orc_entmax_tau_iterative(_ptr(s), s.size, alpha, method, nbins, ftol, wtol,
                                         maxpass, ctypes.byref(tau), ctypes.byref(passes)),
           "entmax_tau_iterative")
    return tau.value, passes.value


# ---------------------------------------------------------- attention level
def attn_fwd(q, k, v, alpha, causal, blk=128, nthreads=0):
    """(o, tau, blk_margin) for [B,H,N,d] inputs; blk_margin is [B,H,T,T]."""
    q, k, v = _d(q), _d(k), _d(v)
    B, H, N, d = q.shape
    T = -(-N // blk) if N else 0
    o = np.zeros_like(q)
    tau = np.zeros((B, H, N))
    marg = np.full((B, H, T, T), -np.inf)
    _check(_L().orc_attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, alpha, int(causal), blk,
                             _ptr(o), _ptr(tau), _ptr(marg), nthreads), "attn_fwd")
    return o, tau, marg


def attn_fwd_rows(q, k, v, alpha, causal, rows, blk=128, nthreads=0):
    """Forward for flat row ids (b*H+h)*N+i: (o_rows [R,d], tau_rows [R], bmax [R,T])."""
    q, k, v = _d(q), _d(k), _d(v)
    B, H, N, d = q.shape
    T = -(-N // blk)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    o = np.zeros((rows.size, d))
    tau = np.zeros(rows.size)
    bmax = np.zeros((rows.size, T))
    _check(_L().orc_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, alpha, int(causal),
                                  blk, _ptr(rows, _i64p), rows.size, _ptr(o), _ptr(tau),
                                  _ptr(bmax), nthreads), "attn_fwd_rows")
    return o, tau, bmax


def attn_otilde_rows(q, k, v, alpha, causal, rows, nthreads=0):
    """otilde_i = sum_j g_ij v_j / sum_j g_ij for flat row ids (b*H+h)*N+i: [R, d]."""
    q, k, v = _d(q), _d(k), _d(v)
    B, H, N, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    ot = np.zeros((rows.size, d))
    _check(_L().orc_attn_otilde_rows(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, alpha, int(causal),
                                     _ptr(rows, _i64p), rows.size, _ptr(ot), nthreads),
           "attn_otilde_rows")
    return ot


def attn_bwd(q, k, v, do, alpha, causal, nthreads=0):
    """(dq, dk, dv, tau, delta) for [B,H,N,d] inputs."""
    q, k, v, do = _d(q), _d(k), _d(v), _d(do)
    B, H, N, d = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    tau = np.zeros((B, H, N))
    delta = np.zeros((B, H, N))
    _check(_L().orc_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B, H, N, d, alpha,
                             int(causal), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(tau), _ptr(delta),
                             nthreads), "attn_bwd")
    return dq, dk, dv, tau, delta


def attn_bwd_head_sampled(qh, kh, vh, doh, alpha, causal, rows, keys, nthreads=0):
    """One head [N,d]: (dq_rows [R,d], dk_keys [K,d], dv_keys [K,d])."""
    qh, kh, vh, doh = _d(qh), _d(kh), _d(vh), _d(doh)
    N, d = qh.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    keys = np.ascontiguousarray(keys, dtype=np.int32)
    dq = np.zeros((rows.size, d))
    dk = np.zeros((keys.size, d))
    dv = np.zeros((keys.size, d))
    _check(_L().orc_attn_bwd_head_sampled(_ptr(qh), _ptr(kh), _ptr(vh), _ptr(doh), N, d, alpha,
                                          int(causal), _ptr(rows, _ip), rows.size,
                                          _ptr(keys, _ip), keys.size, _ptr(dq), _ptr(dk),
                                          _ptr(dv), nthreads), "attn_bwd_head_sampled")
    return dq, dk, dv
