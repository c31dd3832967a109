"""CPU oracle for the Flash PD-SSM recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline
leg may import this package.  The CUDA library never calls it and shares no
code with it.  The arithmetic lives in ``pdssm_oracle.c`` (plain sequential
fp64 C; the selection logits follow the fixed fp32 fmaf-chain contract); this
module only marshals numpy arrays into it.

Sources followed (page title, section):
  * Flash PD-SSM technical summary, Methodology §1 (hard selection: K linear
    scores of u_t, argmax; the chosen matrix is a one-hot column selector, so
    P[pi(j), j] = 1 and memory is O(LN)).
  * Flash PD-SSM technical summary, Methodology §3 (phase A chunk-local
    recurrence, phase B carry scan, phase C carry correction) -- the closed
    PD form of a chunk transfer.
  * Breaking the Memory Wall (PGF), abstract and framework stages -- exact
    analytical derivatives of the SSM by a chunked reverse evolution.

Every function here is pinned by ``tests/test_oracle_pins.py`` against dense
brute force, DFA emulation (Proposition 1), closed forms and finite
differences.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64 = ctypes.c_int64
        p = ctypes.c_void_p
        lib.oracle_select.argtypes = [i64, i64, i64, i64, i64, p, p, p]
        lib.oracle_scan_fwd.argtypes = [i64, i64, i64, i64, i64, p, i64, p,
                                        p, p, p, p, p, p]
        lib.oracle_chunk_transfers.argtypes = [i64, i64, i64, i64, i64, p, i64,
                                               p, p, p, i64, p, p, p]
        lib.oracle_scan_bwd.argtypes = [i64, i64, i64, i64, i64, p, i64, p,
                                        p, p, p, p, p, p, p, p, p, p]
        for f in (lib.oracle_select, lib.oracle_scan_fwd,
                  lib.oracle_chunk_transfers, lib.oracle_scan_bwd):
            f.restype = None
        _LIB = lib
    return _LIB


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _dict_args(pi, H, K, N):
    """pi: [K, N] shared by all heads, or [H, K, N] one per head."""
    pi = _i32(pi)
    if pi.ndim == 2:
        assert pi.shape == (K, N)
        hs = 0
    else:
        assert pi.shape == (H, K, N)
        hs = K * N
    if pi.size and (pi.min() < 0 or pi.max() >= N):
        raise ValueError("dictionary entry outside [0, N)")
    return pi, hs


def _check_k(k, K):
    if k.size and (k.min() < 0 or k.max() >= K):
        raise ValueError("selection index outside [0, K)")


def select(u, W):
    """k[b, h, t] = first argmax_k of the fp32 fmaf chain sum_d W[h,k,d] u[b,t,d].

    u: [B, L, D] float32 (bf16 values already upcast); W: [H, K, D] float32.
    """
    u = np.ascontiguousarray(u, dtype=np.float32)
    W = np.ascontiguousarray(W, dtype=np.float32)
    B, L, D = u.shape
    H, K, D2 = W.shape
    assert D == D2
    k = np.empty((B, H, L), dtype=np.int32)
    _lib().oracle_select(B, L, D, H, K, _ptr(u), _ptr(W), _ptr(k))
    return k


def scan_fwd(pi, k, d, b, c, h0=None):
    """Sequential forward scan; returns (y [B,H,L], h_last [B,H,N]) in fp64."""
    d, b, c = _f64(d), _f64(b), _f64(c)
    B, H, L, N = d.shape
    k = _i32(k)
    assert k.shape == (B, H, L)
    K = pi.shape[-2]
    pi, hs = _dict_args(pi, H, K, N)
    _check_k(k, K)
    h0 = _f64(h0)
    y = np.empty((B, H, L), dtype=np.float64)
    h_last = np.empty((B, H, N), dtype=np.float64)
    _lib().oracle_scan_fwd(B, H, L, N, K, _ptr(pi), hs, _ptr(k), _ptr(d),
                           _ptr(b), _ptr(c), _ptr(h0), _ptr(y), _ptr(h_last))
    return y, h_last


def chunk_transfers(pi, k, d, b, chunk):
    """Closed PD form (Pi int32, Delta fp64, v fp64), each [B, H, C, N]."""
    d, b = _f64(d), _f64(b)
    B, H, L, N = d.shape
    k = _i32(k)
    K = pi.shape[-2]
    pi, hs = _dict_args(pi, H, K, N)
    _check_k(k, K)
    C = (L + chunk - 1) // chunk
    Pi = np.empty((B, H, C, N), dtype=np.int32)
    Delta = np.empty((B, H, C, N), dtype=np.float64)
    v = np.empty((B, H, C, N), dtype=np.float64)
    _lib().oracle_chunk_transfers(B, H, L, N, K, _ptr(pi), hs, _ptr(k),
                                  _ptr(d), _ptr(b), chunk, _ptr(Pi),
                                  _ptr(Delta), _ptr(v))
    return Pi, Delta, v


def scan_bwd(pi, k, d, b, c, h0, g_y, g_hlast=None):
    """Exact adjoint; returns (g_b, g_d, g_c, g_h0) in fp64."""
    d, b, c = _f64(d), _f64(b), _f64(c)
    B, H, L, N = d.shape
    k = _i32(k)
    K = pi.shape[-2]
    pi, hs = _dict_args(pi, H, K, N)
    _check_k(k, K)
    h0, g_y, g_hlast = _f64(h0), _f64(g_y), _f64(g_hlast)
    g_b = np.empty((B, H, L, N), dtype=np.float64)
    g_d = np.empty_like(g_b)
    g_c = np.empty_like(g_b)
    g_h0 = np.empty((B, H, N), dtype=np.float64)
    _lib().oracle_scan_bwd(B, H, L, N, K, _ptr(pi), hs, _ptr(k), _ptr(d),
                           _ptr(b), _ptr(c), _ptr(h0), _ptr(g_y), _ptr(g_hlast),
                           _ptr(g_b), _ptr(g_d), _ptr(g_c), _ptr(g_h0))
    return g_b, g_d, g_c, g_h0
