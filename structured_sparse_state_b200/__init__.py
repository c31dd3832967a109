"""Flash PD-SSM structured-sparse scan on B200 (sm_100a).

Thin Python binding of ``libpdssm.so``: every function here only checks and
marshals PyTorch tensors (device memory, the current stream) into the C ABI
declared in ``include/pdssm.h``; all arithmetic runs in the CUDA kernels.
There is no CPU path: importing this package without the built library, or
calling it with CPU tensors, raises.

    k = pdssm_select(u, W_sel)                          # hard selection
    y, h_last, ws = pdssm_scan_fwd(pi, k, d, b, c, h0, chunk=128, for_bwd=True)
    g_b, g_d, g_c, g_h0 = pdssm_scan_bwd(pi, k, d, b, c, h0, g_y, ws=ws, chunk=128)

Page sources: Flash PD-SSM technical summary, Methodology §1 (hard
selection, one-hot column selector) and §3 (three-phase chunked kernel);
Breaking the Memory Wall (PGF), abstract (exact chunked adjoint).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpdssm.so")

PDSSM_F32, PDSSM_BF16 = 0, 1
STATUS = {0: "PDSSM_OK", 1: "PDSSM_ERR_INVALID_ARG", 2: "PDSSM_ERR_UNSUPPORTED",
          3: "PDSSM_ERR_BAD_INDEX", 4: "PDSSM_ERR_CUDA", 5: "PDSSM_ERR_TIMEOUT",
          6: "PDSSM_ERR_WORKSPACE"}

# every entry point declared in include/pdssm.h
EXPORTS = ("pdssm_status_str", "pdssm_last_error", "pdssm_version",
           "pdssm_workspace_bytes", "pdssm_select", "pdssm_scan_fwd",
           "pdssm_scan_bwd", "pdssm_chunk_transfers", "pdssm_validate",
           "pdssm_ws_status", "pdssm_scan_fwd_noalloc", "pdssm_noalloc_scratch_bytes",
           "pdssm_select_with", "pdssm_select_tc_logits", "pdssm_noalloc_status",
           "pdssm_scan_fwd_traced", "pdssm_scan_bwd_traced", "pdssm_ws_transfers",
           "pdssm_wait_selftest", "pdssm_wait_selftest_ws_bytes", "pdssm_dict_hardmax",
           "pdssm_soft_maps", "pdssm_scan_fwd_maps", "pdssm_surrogate_scratch_bytes",
           "pdssm_surrogate_bwd", "pdssm_select_scan_fwd", "pdssm_scan_fwd_single_pass")

TRACE_MAX_KERNELS = 8

SELECT_METHODS = {"auto": 0, "fma": 1, "tensor_core": 2}


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("L", ctypes.c_int64),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("D_in", ctypes.c_int64)]


class Trace(ctypes.Structure):
    _fields_ = [("events", ctypes.POINTER(ctypes.c_void_p)), ("max_events", ctypes.c_int),
                ("n_kernels", ctypes.c_int), ("names", ctypes.c_char_p * TRACE_MAX_KERNELS)]


class PdssmError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({last_error()})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m structured_sparse_state_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    D = ctypes.POINTER(Dims)
    sig = {
        "pdssm_status_str": (ctypes.c_char_p, [I32]),
        "pdssm_last_error": (ctypes.c_char_p, []),
        "pdssm_version": (I32, []),
        "pdssm_workspace_bytes": (SZ, [D, I64, I64, I32]),
        "pdssm_select": (I32, [D, P, I32, P, P, P]),
        "pdssm_select_with": (I32, [D, P, I32, P, P, I32, P]),
        "pdssm_select_tc_logits": (I32, [D, P, P, P, P, P, P]),
        "pdssm_scan_fwd": (I32, [D, P, I64, P, P, P, P, I32, P, P, P, I64, P, SZ, P]),
        "pdssm_scan_bwd": (I32, [D, P, I64, P, P, P, P, I32, P, P, P, P, P, P, P, I64, P,
                                 SZ, P]),
        "pdssm_chunk_transfers": (I32, [D, P, I64, P, P, P, I32, I64, P, P, P, P, SZ, P]),
        "pdssm_validate": (I32, [D, P, I64, P, P, SZ, P]),
        "pdssm_ws_status": (I32, [P, SZ, P]),
        "pdssm_scan_fwd_noalloc": (I32, [D, P, I64, P, P, P, P, I32, P, P, P, I64, P]),
        "pdssm_noalloc_scratch_bytes": (SZ, []),
        "pdssm_noalloc_status": (I32, [P]),
        "pdssm_ws_transfers": (I32, [D, I64, I64, P, SZ, P, P, P, P, P]),
        "pdssm_wait_selftest": (I32, [I32, I64, P, SZ, P]),
        "pdssm_wait_selftest_ws_bytes": (SZ, []),
        "pdssm_dict_hardmax": (I32, [I64, I64, P, P, P]),
        "pdssm_soft_maps": (I32, [D, P, I32, P, P, I64, ctypes.c_float, P, P]),
        "pdssm_scan_fwd_maps": (I32, [D, P, P, P, P, I32, P, P, P, P]),
        "pdssm_surrogate_scratch_bytes": (SZ, [D, I64]),
        "pdssm_scan_fwd_single_pass": (I32, [D, P, I64, P, P, P, P, I32, P, P, P, I64, P, SZ,
                                             P]),
        "pdssm_select_scan_fwd": (I32, [D, P, I32, P, P, I64, P, P, P, I32, P, P, P, P, I64, P,
                                        SZ, P]),
        "pdssm_surrogate_bwd": (I32, [D, P, I32, P, P, I64, P, P, P, P, I32, P, P, I64, P, SZ,
                                      ctypes.c_float, ctypes.c_float, P, SZ, P, P, P, P]),
        "pdssm_scan_fwd_traced": (I32, [D, P, I64, P, P, P, P, I32, P, P, P, I64, P, SZ, P,
                                        ctypes.POINTER(Trace)]),
        "pdssm_scan_bwd_traced": (I32, [D, P, I64, P, P, P, P, I32, P, P, P, P, P, P, P, I64,
                                        P, SZ, P, ctypes.POINTER(Trace)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


class _Lazy:
    """Loads libpdssm.so on first use, so the build step can import this
    package before the library exists; any call without it raises."""
    _cdll = None

    def __getattr__(self, name):
        if _Lazy._cdll is None:
            _Lazy._cdll = _load()
        return getattr(_Lazy._cdll, name)


_lib = _Lazy()


def lib():
    """The loaded C library (for callers that want the raw ABI)."""
    _lib.pdssm_version        # force the load
    return _Lazy._cdll


def last_error() -> str:
    return (_lib.pdssm_last_error() or b"").decode()


def version() -> int:
    return int(_lib.pdssm_version())


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------
def _check(code: int, what: str):
    if code != 0:
        raise PdssmError(code, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda(t: torch.Tensor, name: str, dtypes) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _dtype_code(t: torch.Tensor) -> int:
    return PDSSM_BF16 if t.dtype == torch.bfloat16 else PDSSM_F32


def _dict_stride(pi: torch.Tensor, H: int, K: int, N: int) -> int:
    if pi.dim() == 2:
        if tuple(pi.shape) != (K, N):
            raise ValueError(f"pi_dict shape {tuple(pi.shape)} != ({K}, {N})")
        return 0
    if tuple(pi.shape) != (H, K, N):
        raise ValueError(f"pi_dict shape {tuple(pi.shape)} != ({H}, {K}, {N})")
    return K * N


def dims(B, H, L, N, K, D_in=0) -> Dims:
    return Dims(int(B), int(H), int(L), int(N), int(K), int(D_in))


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------
def pdssm_workspace_bytes(B, H, L, N, K, chunk, per_head_dict=False, for_bwd=False) -> int:
    dm = dims(B, H, L, N, K)
    n = _lib.pdssm_workspace_bytes(ctypes.byref(dm), K * N if per_head_dict else 0,
                                   int(chunk), int(bool(for_bwd)))
    if n == 0:
        raise PdssmError(1, "pdssm_workspace_bytes")
    return int(n)


def _select_shapes(u, W_sel, k_out):
    _cuda(u, "u", (torch.float32, torch.bfloat16))
    _cuda(W_sel, "W_sel", (torch.float32,))
    B, L, D = u.shape
    H, K, D2 = W_sel.shape
    if D != D2:
        raise ValueError("u and W_sel disagree on D_in")
    if k_out is None:
        k_out = torch.empty((B, H, L), dtype=torch.int32, device=u.device)
    _cuda(k_out, "k_out", (torch.int32,))
    return B, L, D, H, K, k_out


def pdssm_select(u: torch.Tensor, W_sel: torch.Tensor, k_out: Optional[torch.Tensor] = None,
                 stream=None, method: str = "auto") -> torch.Tensor:
    """k[b, h, t] = first argmax_k of the fp32 fma chain sum_q W_sel[h,k,q] u[b,t,q].
    ``method``: "auto" (tensor cores where they apply), "fma" or "tensor_core";
    every route gives the same k bit for bit."""
    B, L, D, H, K, k_out = _select_shapes(u, W_sel, k_out)
    dm = dims(B, H, L, 0, K, D)
    if method == "auto":
        _check(_lib.pdssm_select(ctypes.byref(dm), _ptr(u), _dtype_code(u), _ptr(W_sel),
                                 _ptr(k_out), _stream(stream)), "pdssm_select")
    else:
        _check(_lib.pdssm_select_with(ctypes.byref(dm), _ptr(u), _dtype_code(u), _ptr(W_sel),
                                      _ptr(k_out), SELECT_METHODS[method], _stream(stream)),
               "pdssm_select_with")
    return k_out


def pdssm_select_tc_logits(u: torch.Tensor, W_sel: torch.Tensor, stream=None):
    """Test hook: the tensor-core selection's k, raw logits [B*L, H*K] and
    per-(row, head) scale ||u_row|| * max_k ||W_hk|| (rounded up)."""
    B, L, D, H, K, k_out = _select_shapes(u, W_sel, None)
    logits = torch.empty((B * L, H * K), dtype=torch.float32, device=u.device)
    scale = torch.empty((B * L, H), dtype=torch.float32, device=u.device)
    dm = dims(B, H, L, 0, K, D)
    _check(_lib.pdssm_select_tc_logits(ctypes.byref(dm), _ptr(u), _ptr(W_sel), _ptr(k_out),
                                       _ptr(logits), _ptr(scale), _stream(stream)),
           "pdssm_select_tc_logits")
    return k_out, logits, scale


def _scan_shapes(pi, k, d, b, c):
    _cuda(d, "d", (torch.float32, torch.bfloat16))
    B, H, L, N = d.shape
    for name, t in (("b", b), ("c", c)):
        if t is None:
            continue
        _cuda(t, name, (d.dtype,))
        if t.shape != d.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != d shape {tuple(d.shape)}")
    _cuda(k, "k", (torch.int32,))
    if tuple(k.shape) != (B, H, L):
        raise ValueError("k must be [B, H, L]")
    _cuda(pi, "pi_dict", (torch.int32,))
    K = pi.shape[-2]
    stride = _dict_stride(pi, H, K, N)
    return B, H, L, N, K, stride


def make_workspace(B, H, L, N, K, chunk, device, per_head_dict=False, for_bwd=False):
    n = pdssm_workspace_bytes(B, H, L, N, K, chunk, per_head_dict, for_bwd)
    return torch.empty(n, dtype=torch.uint8, device=device)


def pdssm_scan_fwd(pi_dict, k, d, b, c, h0=None, chunk=128, ws=None, y=None, h_last=None,
                   for_bwd=False, stream=None):
    """Chunked three-phase forward scan; returns (y, h_last, ws)."""
    B, H, L, N, K, stride = _scan_shapes(pi_dict, k, d, b, c)
    dev = d.device
    if ws is None:
        ws = make_workspace(B, H, L, N, K, chunk, dev, stride != 0, for_bwd)
    _cuda(ws, "ws", (torch.uint8,))
    if h0 is not None:
        _cuda(h0, "h0", (torch.float32,))
    if y is None:
        y = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    if h_last is None:
        h_last = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_scan_fwd(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k), _ptr(d),
                               _ptr(b), _ptr(c), _dtype_code(d), _ptr(h0), _ptr(y),
                               _ptr(h_last), int(chunk), _ptr(ws), ws.numel(),
                               _stream(stream)), "pdssm_scan_fwd")
    return y, h_last, ws


def pdssm_scan_fwd_single_pass(pi_dict, k, d, b, c, h0=None, chunk=128, ws=None, y=None,
                               h_last=None, for_bwd=False, stream=None):
    """The forward scan as one kernel (decoupled look-back); same results and
    workspace as pdssm_scan_fwd.  Returns (y, h_last, ws)."""
    B, H, L, N, K, stride = _scan_shapes(pi_dict, k, d, b, c)
    dev = d.device
    if ws is None:
        ws = make_workspace(B, H, L, N, K, chunk, dev, stride != 0, for_bwd)
    _cuda(ws, "ws", (torch.uint8,))
    if h0 is not None:
        _cuda(h0, "h0", (torch.float32,))
    if y is None:
        y = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    if h_last is None:
        h_last = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_scan_fwd_single_pass(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k),
                                           _ptr(d), _ptr(b), _ptr(c), _dtype_code(d), _ptr(h0),
                                           _ptr(y), _ptr(h_last), int(chunk), _ptr(ws),
                                           ws.numel(), _stream(stream)),
           "pdssm_scan_fwd_single_pass")
    return y, h_last, ws


def pdssm_scan_fwd_noalloc(pi_dict, k, d, b, c, h0=None, chunk=128, y=None, h_last=None,
                           stream=None):
    """pdssm_scan_fwd without a workspace argument: for callers that cannot
    allocate device memory, the scratch is the library's fixed device array
    (pdssm_noalloc_scratch_bytes()).  Pass preallocated y / h_last to keep the
    call itself free of allocations.  Returns (y, h_last)."""
    B, H, L, N, K, stride = _scan_shapes(pi_dict, k, d, b, c)
    dev = d.device
    if h0 is not None:
        _cuda(h0, "h0", (torch.float32,))
    if y is None:
        y = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    if h_last is None:
        h_last = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_scan_fwd_noalloc(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k),
                                       _ptr(d), _ptr(b), _ptr(c), _dtype_code(d), _ptr(h0),
                                       _ptr(y), _ptr(h_last), int(chunk), _stream(stream)),
           "pdssm_scan_fwd_noalloc")
    return y, h_last


def pdssm_select_scan_fwd(u, W_sel, pi_dict, d, b, c, h0=None, chunk=128, ws=None, y=None,
                          h_last=None, k_out=None, stream=None):
    """Selection inside the single-pass forward (indices stay in shared
    memory; k_out, if given, receives a copy).  Returns (y, h_last, ws)."""
    _cuda(u, "u", (torch.bfloat16, torch.float32))
    _cuda(W_sel, "W_sel", (torch.float32,))
    _cuda(d, "d", (torch.float32, torch.bfloat16))
    B, H, L, N = d.shape
    Bu, Lu, D = u.shape
    H2, K, D2 = W_sel.shape
    if (Bu, Lu, H2, D2) != (B, L, H, D):
        raise ValueError("u [B, L, D_in] and W_sel [H, K, D_in] disagree with d")
    for name, t in (("b", b), ("c", c)):
        _cuda(t, name, (d.dtype,))
    _cuda(pi_dict, "pi_dict", (torch.int32,))
    stride = _dict_stride(pi_dict, H, K, N)
    dev = d.device
    if ws is None:
        ws = make_workspace(B, H, L, N, K, chunk, dev, stride != 0, False)
    if y is None:
        y = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    if h_last is None:
        h_last = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    if k_out is not None:
        _cuda(k_out, "k_out", (torch.int32,))
    if h0 is not None:
        _cuda(h0, "h0", (torch.float32,))
    dm = dims(B, H, L, N, K, D)
    _check(_lib.pdssm_select_scan_fwd(ctypes.byref(dm), _ptr(u), _dtype_code(u), _ptr(W_sel),
                                      _ptr(pi_dict), stride, _ptr(d), _ptr(b), _ptr(c),
                                      _dtype_code(d), _ptr(h0), _ptr(y), _ptr(h_last),
                                      _ptr(k_out), int(chunk), _ptr(ws), ws.numel(),
                                      _stream(stream)), "pdssm_select_scan_fwd")
    return y, h_last, ws


def pdssm_noalloc_scratch_bytes() -> int:
    return int(_lib.pdssm_noalloc_scratch_bytes())


def pdssm_noalloc_status(stream=None) -> int:
    """Reads and clears the status word of the no-allocation scratch
    (synchronises)."""
    return int(_lib.pdssm_noalloc_status(_stream(stream)))


def pdssm_scan_bwd(pi_dict, k, d, b, c, h0, g_y, ws, chunk=128, g_hlast=None, out=None,
                   stream=None):
    """Exact adjoint; ws must be the forward's (sized with for_bwd=True).
    Returns (g_b, g_d, g_c, g_h0)."""
    B, H, L, N, K, stride = _scan_shapes(pi_dict, k, d, b, c)
    dev = d.device
    _cuda(ws, "ws", (torch.uint8,))
    _cuda(g_y, "g_y", (torch.float32,))
    if h0 is not None:
        _cuda(h0, "h0", (torch.float32,))
    if g_hlast is not None:
        _cuda(g_hlast, "g_hlast", (torch.float32,))
    if out is None:
        out = (torch.empty((B, H, L, N), dtype=torch.float32, device=dev),
               torch.empty((B, H, L, N), dtype=torch.float32, device=dev),
               torch.empty((B, H, L, N), dtype=torch.float32, device=dev),
               torch.empty((B, H, N), dtype=torch.float32, device=dev))
    g_b, g_d, g_c, g_h0 = out
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_scan_bwd(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k), _ptr(d),
                               _ptr(b), _ptr(c), _dtype_code(d), _ptr(h0), _ptr(g_y),
                               _ptr(g_hlast), _ptr(g_b), _ptr(g_d), _ptr(g_c), _ptr(g_h0),
                               int(chunk), _ptr(ws), ws.numel(), _stream(stream)),
           "pdssm_scan_bwd")
    return g_b, g_d, g_c, g_h0


def pdssm_chunk_transfers(pi_dict, k, d, b, chunk, ws=None, stream=None):
    """Phase A transfers (Pi int32, Delta fp32, v fp32), each [B, H, C, N]."""
    B, H, L, N, K, stride = _scan_shapes(pi_dict, k, d, b, None)
    dev = d.device
    C = (L + chunk - 1) // chunk
    if ws is None:
        ws = make_workspace(B, H, L, N, K, chunk, dev, stride != 0)
    Pi = torch.empty((B, H, C, N), dtype=torch.int32, device=dev)
    Dl = torch.empty((B, H, C, N), dtype=torch.float32, device=dev)
    v = torch.empty((B, H, C, N), dtype=torch.float32, device=dev)
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_chunk_transfers(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k),
                                      _ptr(d), _ptr(b), _dtype_code(d), int(chunk), _ptr(Pi),
                                      _ptr(Dl), _ptr(v), _ptr(ws), ws.numel(),
                                      _stream(stream)), "pdssm_chunk_transfers")
    return Pi, Dl, v


def pdssm_ws_transfers(ws, B, H, L, N, K, chunk, per_head_dict=False, stream=None):
    """Test hook: the chunk transfers (Pi, Delta, v) and carries H_c that the
    last forward left in ws, each [B, H, C, N]."""
    _cuda(ws, "ws", (torch.uint8,))
    C = (L + chunk - 1) // chunk
    dev = ws.device
    Pi = torch.empty((B, H, C, N), dtype=torch.int32, device=dev)
    Dl, v, Hc = (torch.empty((B, H, C, N), dtype=torch.float32, device=dev) for _ in range(3))
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_ws_transfers(ctypes.byref(dm), K * N if per_head_dict else 0, int(chunk),
                                   _ptr(ws), ws.numel(), _ptr(Pi), _ptr(Dl), _ptr(v), _ptr(Hc),
                                   _stream(stream)), "pdssm_ws_transfers")
    return Pi, Dl, v, Hc


def pdssm_wait_selftest(which: int, cap_ns: int, device=None, stream=None) -> int:
    """Runs a bounded wait that nothing completes (0: look-back flag, 1:
    mbarrier) with the given cap; returns the status the workspace's status
    word maps to (PDSSM_ERR_TIMEOUT = 5 expected).  Synchronises."""
    n = int(_lib.pdssm_wait_selftest_ws_bytes())
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    _check(_lib.pdssm_wait_selftest(int(which), int(cap_ns), _ptr(ws), n, _stream(stream)),
           "pdssm_wait_selftest")
    return pdssm_ws_status(ws, stream)


def pdssm_validate(pi_dict, k, N, ws=None, stream=None) -> int:
    """Returns the status code (0 = all indices in range).  Synchronises."""
    _cuda(pi_dict, "pi_dict", (torch.int32,))
    _cuda(k, "k", (torch.int32,))
    B, H, L = k.shape
    K = pi_dict.shape[-2]
    stride = _dict_stride(pi_dict, H, K, N)
    if ws is None:
        ws = torch.empty(256, dtype=torch.uint8, device=k.device)
    dm = dims(B, H, L, N, K)
    return int(_lib.pdssm_validate(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k), _ptr(ws),
                                   ws.numel(), _stream(stream)))


def pdssm_ws_status(ws, stream=None) -> int:
    """Reads and clears the workspace status word (synchronises)."""
    _cuda(ws, "ws", (torch.uint8,))
    return int(_lib.pdssm_ws_status(_ptr(ws), ws.numel(), _stream(stream)))


# ----------------------------------------------------------------------------
# kernel-level timing (measurement aid)
# ----------------------------------------------------------------------------
def make_trace_events(n: int = TRACE_MAX_KERNELS + 1, stream=None):
    """n timing events, recorded once so that their CUDA handles exist."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    s = stream or torch.cuda.current_stream()
    for e in evs:
        e.record(s)
    return evs


def _trace_struct(events):
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    tr = Trace()
    tr.events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    tr.max_events = len(events)
    return tr, arr


def _trace_result(tr, events):
    """[(kernel name, ms)] of a finished traced call (synchronise first)."""
    return [(tr.names[i].decode(), events[i].elapsed_time(events[i + 1]))
            for i in range(tr.n_kernels)]


def pdssm_scan_fwd_traced(pi_dict, k, d, b, c, h0, chunk, ws, y, h_last, events, stream=None):
    """pdssm_scan_fwd recording `events` between its kernels; returns a
    function that, after a synchronisation, gives [(kernel, ms)]."""
    B, H, L, N, K, stride = _scan_shapes(pi_dict, k, d, b, c)
    tr, arr = _trace_struct(events)
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_scan_fwd_traced(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k), _ptr(d),
                                      _ptr(b), _ptr(c), _dtype_code(d), _ptr(h0), _ptr(y),
                                      _ptr(h_last), int(chunk), _ptr(ws), ws.numel(),
                                      _stream(stream), ctypes.byref(tr)),
           "pdssm_scan_fwd_traced")
    return lambda: _trace_result(tr, events)


def pdssm_scan_bwd_traced(pi_dict, k, d, b, c, h0, g_y, ws, chunk, out, events, g_hlast=None,
                          stream=None):
    """pdssm_scan_bwd recording `events` between its kernels; returns a
    function that, after a synchronisation, gives [(kernel, ms)]."""
    B, H, L, N, K, stride = _scan_shapes(pi_dict, k, d, b, c)
    tr, arr = _trace_struct(events)
    g_b, g_d, g_c, g_h0 = out
    dm = dims(B, H, L, N, K)
    _check(_lib.pdssm_scan_bwd_traced(ctypes.byref(dm), _ptr(pi_dict), stride, _ptr(k), _ptr(d),
                                      _ptr(b), _ptr(c), _dtype_code(d), _ptr(h0), _ptr(g_y),
                                      _ptr(g_hlast), _ptr(g_b), _ptr(g_d), _ptr(g_c), _ptr(g_h0),
                                      int(chunk), _ptr(ws), ws.numel(), _stream(stream),
                                      ctypes.byref(tr)),
           "pdssm_scan_bwd_traced")
    return lambda: _trace_result(tr, events)


# ----------------------------------------------------------------------------
# dictionary from dense matrices; the original soft selection (comparison)
# ----------------------------------------------------------------------------
def pdssm_dict_hardmax(A: torch.Tensor, stream=None) -> torch.Tensor:
    """pi[..., j] = first argmax_i A[..., i, j] for dense [..., N, N] fp32 A."""
    _cuda(A, "A", (torch.float32,))
    N = A.shape[-1]
    if A.shape[-2] != N:
        raise ValueError("A must be [..., N, N]")
    pi = torch.empty(A.shape[:-1], dtype=torch.int32, device=A.device)
    n = A.numel() // (N * N)
    _check(_lib.pdssm_dict_hardmax(n, N, _ptr(A), _ptr(pi), _stream(stream)),
           "pdssm_dict_hardmax")
    return pi


def pdssm_soft_maps(u, W_sel, A, inv_tau, maps_out=None, stream=None):
    """Per-step column-hardmax maps of the soft-selection mixture (the
    original PD-SSM's transitions); returns int32 [B, H, L, N]."""
    _cuda(u, "u", (torch.float32, torch.bfloat16))
    _cuda(W_sel, "W_sel", (torch.float32,))
    B, L, D = u.shape
    H, K, D2 = W_sel.shape
    if D != D2:
        raise ValueError("u and W_sel disagree on D_in")
    _cuda(A, "A", (torch.float32,))
    N = A.shape[-1]
    if A.dim() == 3:
        a_hs = 0
        if tuple(A.shape) != (K, N, N):
            raise ValueError("A must be [K, N, N] or [H, K, N, N]")
    else:
        a_hs = K * N * N
        if tuple(A.shape) != (H, K, N, N):
            raise ValueError("A must be [K, N, N] or [H, K, N, N]")
    if maps_out is None:
        maps_out = torch.empty((B, H, L, N), dtype=torch.int32, device=u.device)
    _cuda(maps_out, "maps_out", (torch.int32,))
    dm = dims(B, H, L, N, K, D)
    _check(_lib.pdssm_soft_maps(ctypes.byref(dm), _ptr(u), _dtype_code(u), _ptr(W_sel),
                                _ptr(A), a_hs, float(inv_tau), _ptr(maps_out), _stream(stream)),
           "pdssm_soft_maps")
    return maps_out


def pdssm_scan_fwd_maps(maps, d, b, c, h0=None, y=None, h_last=None, stream=None):
    """Forward scan with one map per step; returns (y, h_last)."""
    _cuda(maps, "maps", (torch.int32,))
    _cuda(d, "d", (torch.float32, torch.bfloat16))
    B, H, L, N = d.shape
    if tuple(maps.shape) != (B, H, L, N):
        raise ValueError("maps must be [B, H, L, N]")
    for name, t in (("b", b), ("c", c)):
        _cuda(t, name, (d.dtype,))
        if t.shape != d.shape:
            raise ValueError(f"{name} shape differs from d")
    if h0 is not None:
        _cuda(h0, "h0", (torch.float32,))
    if y is None:
        y = torch.empty((B, H, L), dtype=torch.float32, device=d.device)
    if h_last is None:
        h_last = torch.empty((B, H, N), dtype=torch.float32, device=d.device)
    dm = dims(B, H, L, N, 1)
    _check(_lib.pdssm_scan_fwd_maps(ctypes.byref(dm), _ptr(maps), _ptr(d), _ptr(b), _ptr(c),
                                    _dtype_code(d), _ptr(h0), _ptr(y), _ptr(h_last),
                                    _stream(stream)), "pdssm_scan_fwd_maps")
    return y, h_last


# ----------------------------------------------------------------------------
# straight-through surrogate gradients
# ----------------------------------------------------------------------------
def pdssm_surrogate_bwd(u, W_sel, A, pi_dict, k, d, b, h0, lam, ws, chunk, inv_tau_s,
                        inv_tau_a, stream=None):
    """Surrogate gradients (g_logits [B,H,L,K], g_W like W_sel, g_A like A)
    of the hard model; pi_dict = pdssm_dict_hardmax(A), ws = the forward's
    workspace, lam = g_b of pdssm_scan_bwd.  Allocates its scratch."""
    _cuda(u, "u", (torch.float32, torch.bfloat16))
    _cuda(W_sel, "W_sel", (torch.float32,))
    _cuda(A, "A", (torch.float32,))
    _cuda(lam, "lambda", (torch.float32,))
    _cuda(ws, "ws", (torch.uint8,))
    B, H, L, N, K, _ = _scan_shapes(pi_dict, k, d, b, None)
    D = u.shape[-1]
    a_hs = K * N * N if A.dim() == 4 else 0
    if h0 is not None:
        _cuda(h0, "h0", (torch.float32,))
    dm = dims(B, H, L, N, K, D)
    nbytes = int(_lib.pdssm_surrogate_scratch_bytes(ctypes.byref(dm), a_hs))
    if nbytes == 0:
        raise PdssmError(1, "pdssm_surrogate_scratch_bytes")
    scratch = torch.empty(nbytes, dtype=torch.uint8, device=d.device)
    g_l = torch.empty((B, H, L, K), dtype=torch.float32, device=d.device)
    g_W = torch.empty_like(W_sel)
    g_A = torch.empty_like(A)
    _check(_lib.pdssm_surrogate_bwd(ctypes.byref(dm), _ptr(u), _dtype_code(u), _ptr(W_sel),
                                    _ptr(A), a_hs, _ptr(pi_dict), _ptr(k), _ptr(d), _ptr(b),
                                    _dtype_code(d), _ptr(h0), _ptr(lam), int(chunk), _ptr(ws),
                                    ws.numel(), float(inv_tau_s), float(inv_tau_a),
                                    _ptr(scratch), nbytes, _ptr(g_l), _ptr(g_W), _ptr(g_A),
                                    _stream(stream)), "pdssm_surrogate_bwd")
    return g_l, g_W, g_A
