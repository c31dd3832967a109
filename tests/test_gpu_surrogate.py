"""GPU parity of the straight-through surrogate gradients (Flash PD-SSM
technical summary, Methodology §2) against the oracle: logit, weight and
dictionary gradients within the floored relative error of 1e-5 (fp32
inputs) or 2e-2 (bf16 inputs), after the hard forward and exact adjoint of
the same model run on the GPU."""
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


def _case(seed, B, H, L, N, K, D, per_head, bf16):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((B, L, D)).astype(np.float32)
    W = (rng.standard_normal((H, K, D)) / math.sqrt(D)).astype(np.float32)
    A = rng.standard_normal(((H,) if per_head else ()) + (K, N, N)).astype(np.float32)
    d = rng.uniform(0.5, 1.0, (B, H, L, N)).astype(np.float32)
    b = rng.standard_normal((B, H, L, N)).astype(np.float32)
    c = rng.standard_normal((B, H, L, N)).astype(np.float32)
    h0 = rng.standard_normal((B, H, N)).astype(np.float32)
    g_y = rng.standard_normal((B, H, L)).astype(np.float32)
    if bf16:
        u, d, b, c = (gen.round_bf16(x) for x in (u, d, b, c))
    return u, W, A, d, b, c, h0, g_y


def _run(case, chunk, inv_s, inv_a, bf16):
    u, W, A, d, b, c, h0, g_y = case
    tu, tW, tA = dev(u, bf16=bf16), dev(W), dev(A)
    td, tb, tc = (dev(x, bf16=bf16) for x in (d, b, c))
    th0, tgy = dev(h0), dev(g_y)
    pi = pd.pdssm_dict_hardmax(tA)
    k = pd.pdssm_select(tu, tW)
    y, hl, ws = pd.pdssm_scan_fwd(pi, k, td, tb, tc, th0, chunk=chunk, for_bwd=True)
    g_b, _, _, _ = pd.pdssm_scan_bwd(pi, k, td, tb, tc, th0, tgy, ws, chunk=chunk)
    out = pd.pdssm_surrogate_bwd(tu, tW, tA, pi, k, td, tb, th0, g_b, ws, chunk, inv_s, inv_a)
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws) == 0
    return [x.cpu().numpy() for x in out]


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("N,K,D,chunk", [(8, 4, 16, 16), (32, 8, 64, 64), (64, 16, 128, 128),
                                         (5, 3, 7, 9)])
def test_surrogate_gradients_against_the_oracle(N, K, D, chunk, per_head):
    case = _case(N * 10 + K, 2, 3, 300, N, K, D, per_head, False)
    inv_s, inv_a = 1.5, 2.0
    g_l, g_W, g_A = _run(case, chunk, inv_s, inv_a, False)
    r_l, r_W, r_A = oracle.surrogate_grad(*case[:3], inv_s, inv_a, *case[3:])
    assert floored_relerr(g_l, r_l) <= TOL_F32
    assert floored_relerr(g_W, r_W) <= TOL_F32
    assert floored_relerr(g_A, r_A) <= TOL_F32


def test_surrogate_gradients_bf16_inputs():
    case = _case(77, 1, 4, 500, 64, 16, 128, False, True)
    g_l, g_W, g_A = _run(case, 128, 1.0, 1.0, True)
    r_l, r_W, r_A = oracle.surrogate_grad(*case[:3], 1.0, 1.0, *case[3:])
    for a, r in ((g_l, r_l), (g_W, r_W), (g_A, r_A)):
        assert floored_relerr(a, r) <= TOL_BF16


def test_surrogate_gradients_deterministic():
    case = _case(5, 2, 2, 400, 32, 8, 32, False, False)
    a = _run(case, 64, 1.0, 1.0, False)
    b = _run(case, 64, 1.0, 1.0, False)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
