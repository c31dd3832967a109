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
  * Flash PD-SSM technical summary, Methodology §1 (the original PD-SSM's
    soft selection: a convex combination of dense dictionary matrices, then
    a column hardmax) -- dict_hardmax, soft_maps, scan_fwd_maps.
  * Flash PD-SSM technical summary, Methodology §2 (straight-through
    estimator: hard forward, tempered softmax in the backward, gradients into
    the selection weights and the dictionary matrices) -- surrogate_grad.

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
        f32 = ctypes.c_float
        f64 = ctypes.c_double
        lib.oracle_dict_hardmax.argtypes = [i64, i64, p, p]
        lib.oracle_soft_exp_array.argtypes = [i64, p, p]
        lib.oracle_soft_maps.argtypes = [i64, i64, i64, i64, i64, i64, p, p, p, i64, f32, p]
        lib.oracle_scan_fwd_maps.argtypes = [i64, i64, i64, i64, p, p, p, p, p, p, p]
        lib.oracle_surrogate_grad.argtypes = [i64, i64, i64, i64, i64, i64, p, p, p, i64, f64,
                                              f64, p, p, p, p, p, p, p, p, p]
        for f in (lib.oracle_select, lib.oracle_scan_fwd,
                  lib.oracle_chunk_transfers, lib.oracle_scan_bwd, lib.oracle_dict_hardmax,
                  lib.oracle_soft_exp_array, lib.oracle_soft_maps, lib.oracle_scan_fwd_maps,
                  lib.oracle_surrogate_grad):
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


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def dict_hardmax(A):
    """Column hardmax of dense matrices: pi[..., j] = first argmax_i A[..., i, j].
    A: [..., N, N] float32; returns int32 [..., N]."""
    A = _f32(A)
    N = A.shape[-1]
    assert A.shape[-2] == N
    lead = A.shape[:-2]
    n = int(np.prod(lead)) if lead else 1
    pi = np.empty(lead + (N,), dtype=np.int32)
    _lib().oracle_dict_hardmax(n, N, _ptr(A), _ptr(pi))
    return pi


def soft_exp(x):
    """The fp32 exp of the soft selection (x <= 0), elementwise."""
    x = _f32(x)
    out = np.empty_like(x)
    _lib().oracle_soft_exp_array(x.size, _ptr(x), _ptr(out))
    return out


def soft_maps(u, W, A, inv_tau):
    """Per-step column-hardmax maps of the soft-selection mixture
    sum_k softmax(W u_t * inv_tau)_k A_k.  u: [B, L, D]; W: [H, K, D];
    A: [K, N, N] (shared) or [H, K, N, N]; returns int32 [B, H, L, N]."""
    u, W, A = _f32(u), _f32(W), _f32(A)
    B, L, D = u.shape
    H, K, D2 = W.shape
    assert D == D2
    N = A.shape[-1]
    a_hs = K * N * N if A.ndim == 4 else 0
    maps = np.empty((B, H, L, N), dtype=np.int32)
    _lib().oracle_soft_maps(B, L, D, H, K, N, _ptr(u), _ptr(W), _ptr(A), a_hs,
                            float(np.float32(inv_tau)), _ptr(maps))
    return maps


def scan_fwd_maps(maps, d, b, c, h0=None):
    """Forward scan with one map per step: (y [B,H,L], h_last [B,H,N]) fp64."""
    d, b, c = _f64(d), _f64(b), _f64(c)
    B, H, L, N = d.shape
    maps = _i32(maps)
    assert maps.shape == (B, H, L, N)
    if maps.size and (maps.min() < 0 or maps.max() >= N):
        raise ValueError("map entry outside [0, N)")
    h0 = _f64(h0)
    y = np.empty((B, H, L), dtype=np.float64)
    h_last = np.empty((B, H, N), dtype=np.float64)
    _lib().oracle_scan_fwd_maps(B, H, L, N, _ptr(maps), _ptr(d), _ptr(b), _ptr(c), _ptr(h0),
                                _ptr(y), _ptr(h_last))
    return y, h_last


def surrogate_grad(u, W, A, inv_tau_s, inv_tau_a, d, b, c, h0, g_y, g_hlast=None):
    """Straight-through surrogate gradients (g_l [B,H,L,K], g_W [H,K,D],
    g_A like A) of the hard model whose dictionary is the column hardmax of
    A and whose selection is the argmax of W u_t; see pdssm_oracle.c."""
    u, W, A = _f32(u), _f32(W), _f32(A)
    d, b, c = _f64(d), _f64(b), _f64(c)
    B, H, L, N = d.shape
    H2, K, D = W.shape
    assert H2 == H and u.shape == (B, L, D) and A.shape[-2:] == (N, N)
    a_hs = K * N * N if A.ndim == 4 else 0
    h0, g_y, g_hlast = _f64(h0), _f64(g_y), _f64(g_hlast)
    g_l = np.empty((B, H, L, K), dtype=np.float64)
    g_W = np.empty((H, K, D), dtype=np.float64)
    g_A = np.empty(A.shape, dtype=np.float64)
    _lib().oracle_surrogate_grad(B, H, L, N, K, D, _ptr(u), _ptr(W), _ptr(A), a_hs,
                                 float(inv_tau_s), float(inv_tau_a), _ptr(d), _ptr(b), _ptr(c),
                                 _ptr(h0), _ptr(g_y), _ptr(g_hlast), _ptr(g_l), _ptr(g_W),
                                 _ptr(g_A))
    return g_l, g_W, g_A
