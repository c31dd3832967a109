"""Seeded synthetic inputs for the PD-SSM scan: the five workloads and shrunken
copies of them for tests.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no selection, no scan).  Both the CUDA path and the CPU
oracle read the arrays it returns, so the two sides always see the same bytes.

Every generator uses numpy's PCG64 (``default_rng``) seeded with
``1000 + workload index`` and draws its streams in a fixed order:
dictionary, W_sel, u, d, b, c, h0, k, g_y (absent streams are skipped).
bf16 inputs are rounded to nearest-even and returned as the float32 values of
those bf16 numbers, so the upcast the kernels do is exact.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

# The five workloads.  Sizes, distributions and structure follow the problem
# statement the library is measured on (no public dataset is involved).
WORKLOADS = [
    dict(name="tiny_fp32_select_fwd", B=1, H=1, N=8, K=4, L=256, D_in=16,
         chunk=32, dtype="f32", dict_kind="maps", d_dist=("uniform", 0.5, 1.0),
         b_kind="normal", h0_kind="zero", k_kind="select", grad=False),
    dict(name="fp32_mixed_maps_fwd", B=4, H=8, N=16, K=8, L=4096, D_in=64,
         chunk=64, dtype="f32", dict_kind="perm_then_maps",
         d_dist=("uniform", 0.8, 1.0), b_kind="normal", h0_kind="normal",
         k_kind="select", grad=False),
    dict(name="bf16_select_fwd_N64", B=8, H=16, N=64, K=16, L=16384, D_in=128,
         chunk=128, dtype="bf16", dict_kind="maps", d_dist=("sigmoid", 2.0, 1.0),
         b_kind="normal", h0_kind="zero", k_kind="select", grad=False),
    dict(name="stiff_impulse_fp32_L131072", B=1, H=32, N=32, K=8, L=131072,
         D_in=0, chunk=256, dtype="f32", dict_kind="perm",
         d_dist=("loguniform", 1e-4, 1.0), b_kind="impulse", h0_kind="zero",
         k_kind="uniform", grad=False),
    dict(name="fp32_fwd_bwd_N64_L65536", B=2, H=16, N=64, K=16, L=65536,
         D_in=0, chunk=128, dtype="f32", dict_kind="maps",
         d_dist=("uniform", 0.5, 1.0), b_kind="normal", h0_kind="normal",
         k_kind="uniform", grad=True),
]


def workload(index: int, **overrides) -> dict:
    """A copy of workload ``index`` with some sizes replaced (for tests)."""
    w = dict(WORKLOADS[index])
    w["index"] = index
    w.update(overrides)
    return w


@dataclass
class Inputs:
    cfg: dict
    pi: np.ndarray                      # int32 [K, N] (shared) or [H, K, N]
    d: np.ndarray                       # float32 [B, H, L, N]
    b: np.ndarray
    c: np.ndarray
    W: Optional[np.ndarray] = None      # float32 [H, K, D_in]
    u: Optional[np.ndarray] = None      # float32 [B, L, D_in]
    k: Optional[np.ndarray] = None      # int32 [B, H, L] when given
    h0: Optional[np.ndarray] = None     # float32 [B, H, N] or None (= 0)
    g_y: Optional[np.ndarray] = None    # float32 [B, H, L]
    extra: dict = field(default_factory=dict)

    @property
    def bf16(self) -> bool:
        return self.cfg["dtype"] == "bf16"


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (nearest-even); return them as float32."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def random_perm(rng, N):
    return rng.permutation(N).astype(np.int32)


def random_map(rng, N):
    return rng.integers(0, N, size=N, dtype=np.int64).astype(np.int32)


def random_non_injective_map(rng, N):
    """A uniform random map, drawn again until it is not a permutation."""
    while True:
        m = random_map(rng, N)
        if N == 1 or len(np.unique(m)) < N:
            return m


def make_dictionary(rng, kind: str, K: int, N: int) -> np.ndarray:
    if kind == "maps":
        rows = [random_map(rng, N) for _ in range(K)]
    elif kind == "perm":
        rows = [random_perm(rng, N) for _ in range(K)]
    elif kind == "perm_then_maps":
        rows = [random_perm(rng, N) if kk < K // 2 else
                random_non_injective_map(rng, N) for kk in range(K)]
    else:
        raise ValueError(kind)
    return np.stack(rows).astype(np.int32)


def _draw_d(rng, dist, shape):
    kind, p0, p1 = dist
    if kind == "uniform":
        return (p0 + (p1 - p0) * rng.random(shape, dtype=np.float32)).astype(np.float32)
    if kind == "loguniform":
        lo, hi = math.log(p0), math.log(p1)
        e = rng.random(shape, dtype=np.float64)
        return np.exp(lo + (hi - lo) * e).astype(np.float32)
    if kind == "sigmoid":            # d = sigmoid(z), z ~ N(p0, p1^2), host fp64
        z = p0 + p1 * rng.standard_normal(shape, dtype=np.float64)
        return (1.0 / (1.0 + np.exp(-z))).astype(np.float32)
    raise ValueError(kind)


def generate(cfg: dict, seed: Optional[int] = None) -> Inputs:
    """Draw one workload's inputs.  ``cfg`` comes from :func:`workload`."""
    if seed is None:
        seed = 1000 + int(cfg.get("index", 0))
    rng = np.random.default_rng(seed)
    B, H, N, K, L = cfg["B"], cfg["H"], cfg["N"], cfg["K"], cfg["L"]
    D_in = cfg.get("D_in", 0)
    bf16 = cfg["dtype"] == "bf16"
    rb = round_bf16 if bf16 else (lambda a: a)
    shape = (B, H, L, N)

    pi = make_dictionary(rng, cfg["dict_kind"], K, N)
    W = u = k = h0 = g_y = None
    if cfg["k_kind"] == "select":
        W = (rng.standard_normal((H, K, D_in), dtype=np.float32)
             / np.float32(math.sqrt(D_in))).astype(np.float32)
        u = rb(rng.standard_normal((B, L, D_in), dtype=np.float32))
    d = rb(_draw_d(rng, cfg["d_dist"], shape))
    if cfg["b_kind"] == "normal":
        b = rb(rng.standard_normal(shape, dtype=np.float32))
    elif cfg["b_kind"] == "impulse":       # b_0 = e_0 on every (b, h), else 0
        b = np.zeros(shape, dtype=np.float32)
        if L > 0:
            b[:, :, 0, 0] = 1.0
    else:
        raise ValueError(cfg["b_kind"])
    c = rb(rng.standard_normal(shape, dtype=np.float32))
    if cfg["h0_kind"] == "normal":
        h0 = rng.standard_normal((B, H, N), dtype=np.float32)
    if cfg["k_kind"] == "uniform":
        k = rng.integers(0, K, size=(B, H, L), dtype=np.int64).astype(np.int32)
    if cfg.get("grad"):
        g_y = rng.standard_normal((B, H, L), dtype=np.float32)
    return Inputs(cfg=cfg, pi=pi, d=d, b=b, c=c, W=W, u=u, k=k, h0=h0, g_y=g_y)


def with_fields(inp: Inputs, **kw) -> Inputs:
    return replace(inp, **kw)
