"""pdssm_scan_fwd_noalloc: the forward scan for callers that cannot allocate
device memory (an allocator owned by someone else, a loop where cudaMalloc
would synchronise the device, no allocation allowed after start-up).  Its
scratch is a fixed device array inside the library, so the caller passes
only inputs and outputs.

Collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.  It must pass alone in a fresh
process as well as after the other tests (the shared array keeps whatever
an earlier call left in it)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import pdssm_inputs as gen
import structured_sparse_state_b200 as pd
from parity_util import floored_relerr, to_device, tol_for


def _noalloc_raw(t, inp, chunk, y, h_last):
    """Call the entry point through the C ABI with ctypes, no binding helper."""
    B, H, L, N = inp.d.shape
    K = inp.pi.shape[-2]
    dm = pd.dims(B, H, L, N, K)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda x: None if x is None else ctypes.c_void_p(x.data_ptr())
    stride = K * N if inp.pi.ndim == 3 else 0
    return pd.lib().pdssm_scan_fwd_noalloc(
        ctypes.byref(dm), ptr(t["pi"]), stride, ptr(t["k"]), ptr(t["d"]), ptr(t["b"]),
        ptr(t["c"]), pd.PDSSM_BF16 if inp.bf16 else pd.PDSSM_F32, ptr(t["h0"]), ptr(y),
        ptr(h_last), chunk, stream)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cases = [(gen.workload(4, B=1, H=2, L=3000), 128),          # fp32, N = 64, h0 given
             (gen.workload(2, B=1, H=3, L=1000, k_kind="uniform"), 128)]   # bf16, h0 = 0
    for cfg, chunk in cases:
        inp = gen.generate(cfg)
        if inp.k is None:
            inp.k = np.random.default_rng(5).integers(0, cfg["K"], size=inp.d.shape[:3]).astype(np.int32)
        t = to_device(inp)
        t["k"] = torch.from_numpy(inp.k).cuda()
        B, H, L, N = inp.d.shape
        assert pd.pdssm_workspace_bytes(B, H, L, N, cfg["K"], chunk) <= \
            pd.pdssm_noalloc_scratch_bytes()
        y_ref, hl_ref, _ = pd.pdssm_scan_fwd(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"],
                                             chunk=chunk)
        y = torch.empty_like(y_ref)
        hl = torch.empty_like(hl_ref)
        assert _noalloc_raw(t, inp, chunk, y, hl) == 0, pd.last_error()
        torch.cuda.synchronize()
        tol = tol_for(inp)
        assert floored_relerr(y.cpu().numpy(), y_ref.cpu().numpy()) <= tol
        assert floored_relerr(hl.cpu().numpy(), hl_ref.cpu().numpy()) <= tol
        assert pd.pdssm_noalloc_status() == 0


@pytest.mark.gpu
def test_noalloc_per_head_dictionary_against_the_oracle():
    """One dictionary per head (a larger workspace through the same size
    check), compared with the oracle itself on two calls in a row."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cfg = gen.workload(1, B=2, H=4, L=700)
    inp = gen.generate(cfg)
    rng = np.random.default_rng(31)
    H, K, N = 4, cfg["K"], cfg["N"]
    inp.pi = rng.integers(0, N, size=(H, K, N)).astype(np.int32)
    t = to_device(inp)
    k_np = inp.k if inp.k is not None else oracle.select(inp.u, inp.W)
    t["k"] = torch.from_numpy(np.ascontiguousarray(k_np)).cuda()
    y_ref, hl_ref = oracle.scan_fwd(inp.pi, k_np, inp.d, inp.b, inp.c, inp.h0)
    for _ in range(2):
        y = torch.full(y_ref.shape, float("nan"), dtype=torch.float32, device="cuda")
        hl = torch.full(hl_ref.shape, float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_raw(t, inp, 64, y, hl) == 0, pd.last_error()
        assert pd.pdssm_noalloc_status() == 0
        assert floored_relerr(y.cpu().numpy(), y_ref) <= tol_for(inp)
        assert floored_relerr(hl.cpu().numpy(), hl_ref) <= tol_for(inp)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Requests whose workspace would not fit the fixed array are refused
    before anything is launched."""
    big = pd.dims(64, 64, 1 << 16, 64, 16)
    P = ctypes.c_void_p(256)
    st = pd.lib().pdssm_scan_fwd_noalloc(ctypes.byref(big), P, 0, P, P, P, P, 0, None, P, None,
                                         128, None)
    assert st == 2   # PDSSM_ERR_UNSUPPORTED
    assert "exceeds the static scratch" in pd.last_error()
    assert pd.pdssm_noalloc_scratch_bytes() == 4 << 20
    # shapes beyond the library's limits get the same status as pdssm_scan_fwd
    wide = pd.dims(1, 1, 16, 65, 4)
    st = pd.lib().pdssm_scan_fwd_noalloc(ctypes.byref(wide), P, 0, P, P, P, P, 0, None, P, None,
                                         16, None)
    assert st == 2 and "N > 64" in pd.last_error()
