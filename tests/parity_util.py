"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the C ABI binding, run the oracle, compare."""
import numpy as np
import torch

import oracle

TOL_F32 = 1e-5
TOL_BF16 = 2e-2


def floored_relerr(a, r):
    """max_i |a_i - r_i| / max(|r_i|, rms(r)): relative error for typical and
    large entries, rms-scaled absolute error near zero."""
    a = np.asarray(a, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    if r.size == 0:
        return 0.0
    assert np.isfinite(a).all(), "non-finite value in the CUDA output"
    rms = float(np.sqrt(np.mean(r * r)))
    floor = np.maximum(np.abs(r), max(rms, 1e-300))
    return float(np.max(np.abs(a - r) / floor))


def tol_for(inp):
    return TOL_BF16 if inp.bf16 else TOL_F32


def dev(x, dtype=torch.float32, bf16=False):
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x))
    if bf16:
        t = t.to(torch.bfloat16)            # exact: values are already bf16
    elif t.dtype != dtype:
        t = t.to(dtype)
    return t.cuda()


def to_device(inp):
    bf = inp.bf16
    out = dict(
        pi=dev(inp.pi, torch.int32),
        d=dev(inp.d, bf16=bf), b=dev(inp.b, bf16=bf), c=dev(inp.c, bf16=bf),
        h0=dev(inp.h0), g_y=dev(inp.g_y),
        k=dev(inp.k, torch.int32) if inp.k is not None else None,
        W=dev(inp.W), u=dev(inp.u, bf16=bf) if inp.u is not None else None)
    return out


def oracle_k(inp):
    return inp.k if inp.k is not None else oracle.select(inp.u, inp.W)


def sample_rows(B, H, n, seed=0):
    rng = np.random.default_rng(seed)
    pairs = [(int(rng.integers(0, B)), int(rng.integers(0, H))) for _ in range(n)]
    return sorted(set(pairs))
