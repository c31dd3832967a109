"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point its header declares, sizes workspaces, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import pytest

import structured_sparse_state_b200 as pd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pdssm_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "pdssm_scan_fwd" in names and "pdssm_select" in names
    lib = ctypes.CDLL(pd.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(pd.EXPORTS) <= set(names)


def test_status_strings_and_version():
    assert pd.lib().pdssm_status_str(0) == b"PDSSM_OK"
    assert pd.lib().pdssm_status_str(5) == b"PDSSM_ERR_TIMEOUT"
    assert pd.lib().pdssm_status_str(99) == b"PDSSM_ERR_UNKNOWN"
    assert pd.version() >= 100


def test_workspace_bytes_grows_with_carries_and_backward():
    a = pd.pdssm_workspace_bytes(2, 4, 1000, 32, 8, 128)
    b = pd.pdssm_workspace_bytes(2, 4, 1000, 32, 8, 64)
    c = pd.pdssm_workspace_bytes(2, 4, 1000, 32, 8, 128, for_bwd=True)
    d = pd.pdssm_workspace_bytes(2, 4, 1000, 32, 8, 128, per_head_dict=True)
    assert 0 < a < b and a < c and a < d
    # O(B*H*ceil(L/chunk)*N): carries are 1/chunk of the size of d
    C = -(-1000 // 128)
    assert a >= 4 * 2 * 4 * C * 32 * 4
    assert a < 2 * 4 * 1000 * 32 * 4


@pytest.mark.parametrize("bad,code", [
    (dict(N=0), 1), (dict(N=65), 2), (dict(K=0), 1), (dict(K=33), 2),
    (dict(B=0), 1), (dict(L=-1), 1)])
def test_scan_rejects_bad_sizes_before_launch(bad, code):
    kw = dict(B=1, H=1, L=10, N=8, K=4)
    kw.update(bad)
    dm = pd.dims(**kw)
    st = pd.lib().pdssm_scan_fwd(ctypes.byref(dm), ctypes.c_void_p(256), 0, ctypes.c_void_p(256),
                                 ctypes.c_void_p(256), ctypes.c_void_p(256),
                                 ctypes.c_void_p(256), 0, None, ctypes.c_void_p(256), None, 4,
                                 ctypes.c_void_p(256), 1 << 20, None)
    assert st == code
    assert pd.last_error() != ""


def test_scan_rejects_small_workspace_and_null_pointers():
    dm = pd.dims(1, 1, 10, 8, 4)
    P = ctypes.c_void_p(256)
    st = pd.lib().pdssm_scan_fwd(ctypes.byref(dm), P, 0, P, P, P, P, 0, None, P, None, 4, P, 16,
                                 None)
    assert st == 6                       # PDSSM_ERR_WORKSPACE
    st = pd.lib().pdssm_scan_fwd(ctypes.byref(dm), P, 0, None, P, P, P, 0, None, P, None, 4, P,
                                 1 << 20, None)
    assert st == 1                       # NULL k
    st = pd.lib().pdssm_scan_fwd(ctypes.byref(dm), P, 0, P, P, P, P, 0, None, P, None, 0, P,
                                 1 << 20, None)
    assert st == 1                       # chunk = 0
    st = pd.lib().pdssm_scan_fwd(ctypes.byref(dm), P, 0, P, P, P, P, 7, None, P, None, 4, P,
                                 1 << 20, None)
    assert st == 1                       # unknown dtype
    st = pd.lib().pdssm_scan_fwd(ctypes.byref(dm), P, 0, P, P, P, P, 0, None, P, None, 4,
                                 ctypes.c_void_p(260), 1 << 20, None)
    assert st == 1                       # misaligned workspace


def test_backward_rejects_long_chunks():
    dm = pd.dims(1, 1, 1000, 8, 4)
    P = ctypes.c_void_p(256)
    st = pd.lib().pdssm_scan_bwd(ctypes.byref(dm), P, 0, P, P, P, P, 0, None, P, None, P, P, P,
                                 None, 512, P, 1 << 30, None)
    assert st == 2


def test_select_rejects_bad_sizes():
    P = ctypes.c_void_p(256)
    for kw, code in ((dict(K=33, D_in=4), 2), (dict(K=4, D_in=0), 1), (dict(K=4, D_in=300), 2)):
        dm = pd.dims(1, 1, 10, 0, kw["K"], kw["D_in"])
        assert pd.lib().pdssm_select(ctypes.byref(dm), P, 0, P, P, None) == code


def test_binding_refuses_cpu_tensors():
    import torch
    u = torch.zeros(1, 4, 8)
    W = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        pd.pdssm_select(u, W)


def test_select_with_rejects_an_unknown_method():
    dm = pd.dims(1, 1, 10, 0, 4, 16)
    P = ctypes.c_void_p(256)
    st = pd.lib().pdssm_select_with(ctypes.byref(dm), P, 0, P, P, 7, None)
    assert st == 1 and "unknown selection method" in pd.last_error()


def test_traced_calls_need_a_trace_with_two_events():
    dm = pd.dims(1, 1, 10, 8, 4)
    P = ctypes.c_void_p(256)
    lib = pd.lib()
    assert lib.pdssm_scan_fwd_traced(ctypes.byref(dm), P, 0, P, P, P, P, 0, None, P, None, 4,
                                     P, 1 << 20, None, None) == 1
    ev = (ctypes.c_void_p * 1)(None)
    tr = pd.Trace()
    tr.events = ctypes.cast(ev, ctypes.POINTER(ctypes.c_void_p))
    tr.max_events = 1
    assert lib.pdssm_scan_fwd_traced(ctypes.byref(dm), P, 0, P, P, P, P, 0, None, P, None, 4,
                                     P, 1 << 20, None, ctypes.byref(tr)) == 1
    assert "two events" in pd.last_error()
