"""GPU parity of the selection inside the single-pass forward
(pdssm_select_scan_fwd): the indices each CTA computes for its own chunk
(warp-level bf16 tensor-core logits, certified argmax, exact fma chains near
ties) must equal the oracle's selection bit for bit, and y / h_last must
match the oracle within 2e-2 (bf16 inputs) or 1e-5 (fp32 d, b, c)."""
import math

import numpy as np
import pytest
import torch

import oracle
import pdssm_inputs as gen
import structured_sparse_state_b200 as pd
from parity_util import TOL_BF16, TOL_F32, dev, floored_relerr, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _run(u, W, pi, d, b, c, h0, chunk, bf16_in):
    B, H, L, N = d.shape
    k_out = torch.full((B, H, L), -7, dtype=torch.int32, device="cuda")
    y, hl, ws = pd.pdssm_select_scan_fwd(dev(u, bf16=True), dev(W), dev(pi, torch.int32),
                                         dev(d, bf16=bf16_in), dev(b, bf16=bf16_in),
                                         dev(c, bf16=bf16_in), dev(h0), chunk=chunk, k_out=k_out)
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws) == 0
    return y.cpu().numpy(), hl.cpu().numpy(), k_out.cpu().numpy()


@pytest.mark.parametrize("idx,over", [(2, dict(B=2, H=3, L=1000)), (2, dict(B=1, H=16, L=300)),
                                      (1, dict(B=2, H=4, L=777)), (0, {})])
def test_fused_selection_workloads(idx, over):
    inp = gen.generate(gen.workload(idx, **over))
    u = gen.round_bf16(inp.u)
    if inp.cfg["N"] not in (32, 64):
        pytest.skip("the single-pass forward serves N = 32 and 64")
    y, hl, k = _run(u, inp.W, inp.pi, inp.d, inp.b, inp.c, inp.h0, inp.cfg["chunk"], inp.bf16)
    kr = oracle.select(u, inp.W)
    assert (k == kr).all()
    yr, hlr = oracle.scan_fwd(inp.pi, kr, inp.d, inp.b, inp.c, inp.h0)
    tol = TOL_BF16 if inp.bf16 else TOL_F32
    assert floored_relerr(y, yr) <= tol and floored_relerr(hl, hlr) <= tol


@pytest.mark.parametrize("K,D,chunk,N", [(1, 16, 16, 32), (4, 64, 64, 64), (8, 48, 129, 32),
                                         (16, 128, 128, 64), (16, 256, 1000, 64), (5, 32, 7, 32),
                                         (13, 80, 300, 64)])
def test_fused_selection_shapes(K, D, chunk, N):
    rng = np.random.default_rng(K * 100 + D)
    B, H, L = 2, 3, 901
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    W = (rng.standard_normal((H, K, D)) / math.sqrt(D)).astype(np.float32)
    pi = rng.integers(0, N, size=(K, N)).astype(np.int32)
    d = rng.uniform(0.5, 1, (B, H, L, N)).astype(np.float32)
    b = rng.standard_normal((B, H, L, N)).astype(np.float32)
    c = rng.standard_normal((B, H, L, N)).astype(np.float32)
    h0 = rng.standard_normal((B, H, N)).astype(np.float32)
    y, hl, k = _run(u, W, pi, d, b, c, h0, chunk, False)
    kr = oracle.select(u, W)
    assert (k == kr).all()
    yr, hlr = oracle.scan_fwd(pi, kr, d, b, c, h0)
    assert floored_relerr(y, yr) <= TOL_F32 and floored_relerr(hl, hlr) <= TOL_F32


def test_fused_selection_near_ties_and_duplicates():
    """Rows of W that differ by ~1e-6 (most decisions go to the exact
    chains) and exact duplicate rows (the first index wins)."""
    rng = np.random.default_rng(77)
    H, K, D, B, L, N = 4, 16, 128, 1, 512, 64
    base = (rng.standard_normal((H, 1, D)) / np.sqrt(D)).astype(np.float32)
    W = (base + 1e-6 * rng.standard_normal((H, K, D))).astype(np.float32)
    W[:, 5] = W[:, 3]
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    pi = rng.integers(0, N, size=(K, N)).astype(np.int32)
    d = rng.uniform(0.5, 1, (B, H, L, N)).astype(np.float32)
    b = rng.standard_normal((B, H, L, N)).astype(np.float32)
    c = rng.standard_normal((B, H, L, N)).astype(np.float32)
    _, _, k = _run(u, W, pi, d, b, c, None, 128, False)
    assert (k == oracle.select(u, W)).all()


def test_fused_selection_gaps_just_above_the_certification_threshold():
    """Top-2 gaps in [2.4, 3.6] x the certification half-width: decided by
    the single-candidate branch, still bit-exact."""
    H, K, D, B, L, N = 4, 16, 128, 2, 2048, 64
    rng = np.random.default_rng(909)
    W = (rng.standard_normal((H, 1, D)) / np.sqrt(D)).astype(np.float32).repeat(K, 1)
    W[:, 1, 0] -= 1.0
    W[:, 2:, 1] -= 0.5
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    u[:, :, 1] = 4.0
    ceps = 1.01 * (D * 2.0 ** -21 + 2.0 ** -16 + D * 2.0 ** -24)
    wn = np.sqrt((W.astype(np.float64) ** 2).sum(2)).max()
    target = rng.uniform(2.4, 3.6, (B, L)) * np.where(rng.random((B, L)) < 0.5, 1.0, -1.0)
    for _ in range(3):
        un = np.sqrt((u.astype(np.float64) ** 2).sum(2))
        u[:, :, 0] = target * ceps * un * wn * 1.002
        u = gen.round_bf16(u)
    pi = rng.integers(0, N, size=(K, N)).astype(np.int32)
    d = np.full((B, H, L, N), 0.9, np.float32)
    b = rng.standard_normal((B, H, L, N)).astype(np.float32)
    c = rng.standard_normal((B, H, L, N)).astype(np.float32)
    _, _, k = _run(u, W, pi, d, b, c, None, 128, False)
    kr = oracle.select(u, W)
    assert (k == kr).all() and set(np.unique(kr)) == {0, 1}


def test_fused_selection_rejects_unsupported_shapes():
    rng = np.random.default_rng(1)
    d = torch.rand(1, 2, 64, 64, device="cuda")
    pi = torch.zeros(32, 64, dtype=torch.int32, device="cuda")
    u = torch.randn(1, 64, 32, device="cuda").to(torch.bfloat16)
    W = torch.randn(2, 32, 32, device="cuda")
    with pytest.raises(pd.PdssmError):           # K = 32
        pd.pdssm_select_scan_fwd(u, W, pi, d, d, d, chunk=16)
    with pytest.raises(pd.PdssmError):           # chunk > 1024
        pd.pdssm_select_scan_fwd(u, W[:, :8].contiguous(), pi[:8].contiguous(), d, d, d,
                                 chunk=2048)
    with pytest.raises(pd.PdssmError):           # fp32 u
        pd.pdssm_select_scan_fwd(u.float(), W[:, :8].contiguous(), pi[:8].contiguous(), d, d, d,
                                 chunk=16)


def test_fused_selection_full_size_equals_the_two_calls():
    """The full bf16 selection workload: indices equal the standalone
    selection's on every (b, h, t); y and h_last equal the two-call path's
    within the bf16 tolerance; sampled rows against the oracle."""
    cfg = gen.workload(2)
    inp = gen.generate(cfg)
    u, W = dev(inp.u, bf16=True), dev(inp.W)
    pi = dev(inp.pi, torch.int32)
    d, b, c = (dev(x, bf16=True) for x in (inp.d, inp.b, inp.c))
    k_sep = pd.pdssm_select(u, W)
    y_sep, hl_sep, _ = pd.pdssm_scan_fwd(pi, k_sep, d, b, c, None, chunk=cfg["chunk"])
    k_f = torch.empty_like(k_sep)
    y_f, hl_f, ws = pd.pdssm_select_scan_fwd(u, W, pi, d, b, c, None, chunk=cfg["chunk"],
                                             k_out=k_f)
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws) == 0
    assert torch.equal(k_f, k_sep)
    assert floored_relerr(y_f.cpu().numpy(), y_sep.cpu().numpy()) <= 1e-5
    assert floored_relerr(hl_f.cpu().numpy(), hl_sep.cpu().numpy()) <= 1e-5
    for bb, hh in sample_rows(cfg["B"], cfg["H"], 3, seed=9):
        kr = oracle.select(inp.u[bb:bb + 1], inp.W[hh:hh + 1])
        yr, hlr = oracle.scan_fwd(inp.pi, kr, inp.d[bb:bb + 1, hh:hh + 1],
                                  inp.b[bb:bb + 1, hh:hh + 1], inp.c[bb:bb + 1, hh:hh + 1], None)
        assert floored_relerr(y_f[bb, hh].cpu().numpy(), yr[0, 0]) <= TOL_BF16
