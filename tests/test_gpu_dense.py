"""GPU parity of the dictionary-from-dense-matrices and soft-selection
kernels (Flash PD-SSM technical summary, Methodology §1) against the CPU
oracle: the column-hardmax dictionary and the per-step soft-selection maps
bit for bit (integer decisions taken in the same fixed fp32 arithmetic on
both sides), the per-step-map scan within the floored relative error of
1e-5 (fp32 inputs) or 2e-2 (bf16 inputs)."""
import math

import numpy as np
import pytest
import torch

import oracle
import pdssm_inputs as gen
import structured_sparse_state_b200 as pd
from parity_util import TOL_BF16, TOL_F32, dev, floored_relerr

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("N", [1, 7, 32, 64])
def test_dict_hardmax_bit_exact(N):
    rng = np.random.default_rng(N)
    A = rng.standard_normal((3, 16, N, N)).astype(np.float32)
    A[0, 0, :, 0] = 2.0                      # a whole tied column: row 0 wins
    if N > 3:
        A[1, 2, 1, 3] = A[1, 2, 3, 3] = 9.0  # a two-way tie: row 1 wins
    pi = pd.pdssm_dict_hardmax(dev(A)).cpu().numpy()
    assert (pi == oracle.dict_hardmax(A)).all()


def _soft_inputs(seed, B, H, L, D, K, N, per_head, bf16):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((B, L, D)).astype(np.float32)
    if bf16:
        u = gen.round_bf16(u)
    W = (rng.standard_normal((H, K, D)) / math.sqrt(D)).astype(np.float32)
    A = rng.standard_normal(((H,) if per_head else ()) + (K, N, N)).astype(np.float32)
    return u, W, A


@pytest.mark.parametrize("inv_tau", [0.25, 1.0, 7.0, 1e6])
@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("per_head", [False, True])
def test_soft_maps_bit_exact(inv_tau, bf16, per_head):
    u, W, A = _soft_inputs(11, 2, 3, 53, 40, 6, 24, per_head, bf16)
    maps = pd.pdssm_soft_maps(dev(u, bf16=bf16), dev(W), dev(A), inv_tau).cpu().numpy()
    assert (maps == oracle.soft_maps(u, W, A, inv_tau)).all()


@pytest.mark.parametrize("K,N,D", [(1, 8, 16), (16, 64, 128), (32, 32, 64), (5, 3, 7)])
def test_soft_maps_shapes_bit_exact(K, N, D):
    u, W, A = _soft_inputs(K * N + D, 1, 2, 40, D, K, N, False, True)
    maps = pd.pdssm_soft_maps(dev(u, bf16=True), dev(W), dev(A), 1.0).cpu().numpy()
    assert (maps == oracle.soft_maps(u, W, A, 1.0)).all()


@pytest.mark.parametrize("N", [1, 7, 32, 33, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_scan_fwd_maps_against_the_oracle(N, dtype):
    rng = np.random.default_rng(N + 100)
    B, H, L = 2, 3, 300
    maps = rng.integers(0, N, size=(B, H, L, N)).astype(np.int32)
    d = rng.uniform(0.5, 1.0, (B, H, L, N)).astype(np.float32)
    b = rng.standard_normal((B, H, L, N)).astype(np.float32)
    c = rng.standard_normal((B, H, L, N)).astype(np.float32)
    h0 = rng.standard_normal((B, H, N)).astype(np.float32)
    bf = dtype == "bf16"
    if bf:
        d, b, c = (gen.round_bf16(x) for x in (d, b, c))
    y, hl = pd.pdssm_scan_fwd_maps(dev(maps, torch.int32), dev(d, bf16=bf), dev(b, bf16=bf),
                                   dev(c, bf16=bf), dev(h0))
    y_r, hl_r = oracle.scan_fwd_maps(maps, d, b, c, h0)
    tol = TOL_BF16 if bf else TOL_F32
    assert floored_relerr(y.cpu().numpy(), y_r) <= tol
    assert floored_relerr(hl.cpu().numpy(), hl_r) <= tol


def test_scan_fwd_maps_empty_sequence_returns_h0():
    h0 = torch.randn(1, 2, 8, device="cuda")
    d = torch.empty((1, 2, 0, 8), device="cuda")
    maps = torch.empty((1, 2, 0, 8), dtype=torch.int32, device="cuda")
    y, hl = pd.pdssm_scan_fwd_maps(maps, d, d, d, h0)
    assert torch.equal(hl, h0) and y.numel() == 0


def test_soft_selection_path_end_to_end():
    """The original PD-SSM forward (soft maps, then the per-step-map scan)
    against the oracle's, at a reduced copy of the bf16 selection workload."""
    cfg = gen.workload(2, B=1, H=4, L=400)
    inp = gen.generate(cfg)
    rng = np.random.default_rng(3)
    A = rng.standard_normal((cfg["K"], cfg["N"], cfg["N"])).astype(np.float32)
    maps = pd.pdssm_soft_maps(dev(inp.u, bf16=True), dev(inp.W), dev(A), 1.0)
    maps_r = oracle.soft_maps(inp.u, inp.W, A, 1.0)
    assert (maps.cpu().numpy() == maps_r).all()
    y, hl = pd.pdssm_scan_fwd_maps(maps, dev(inp.d, bf16=True), dev(inp.b, bf16=True),
                                   dev(inp.c, bf16=True))
    y_r, hl_r = oracle.scan_fwd_maps(maps_r, inp.d, inp.b, inp.c)
    assert floored_relerr(y.cpu().numpy(), y_r) <= TOL_BF16
    assert floored_relerr(hl.cpu().numpy(), hl_r) <= TOL_BF16


def test_flash_path_with_a_dictionary_from_dense_matrices():
    """Hard selection over the column-hardmax dictionary of dense matrices:
    dictionary bit-exact, then the Flash scan against the oracle."""
    cfg = gen.workload(2, B=1, H=2, L=500)
    inp = gen.generate(cfg)
    rng = np.random.default_rng(4)
    A = rng.standard_normal((cfg["K"], cfg["N"], cfg["N"])).astype(np.float32)
    pi = pd.pdssm_dict_hardmax(dev(A))
    pi_r = oracle.dict_hardmax(A)
    assert (pi.cpu().numpy() == pi_r).all()
    k = pd.pdssm_select(dev(inp.u, bf16=True), dev(inp.W))
    y, hl, ws = pd.pdssm_scan_fwd(pi, k, dev(inp.d, bf16=True), dev(inp.b, bf16=True),
                                  dev(inp.c, bf16=True), None, chunk=cfg["chunk"])
    k_r = oracle.select(inp.u, inp.W)
    assert (k.cpu().numpy() == k_r).all()
    y_r, hl_r = oracle.scan_fwd(pi_r, k_r, inp.d, inp.b, inp.c, None)
    assert floored_relerr(y.cpu().numpy(), y_r) <= TOL_BF16
    assert floored_relerr(hl.cpu().numpy(), hl_r) <= TOL_BF16
