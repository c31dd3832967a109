"""GPU checks of the multi-head layer wrapper (Flash PD-SSM technical
summary, Methodology §4): the autograd function's forward, exact adjoint and
surrogate gradients against the oracle, and a pre-norm layer that trains
end to end through the library."""
import math

import numpy as np
import pytest
import torch

import oracle
import pdssm_inputs as gen
from parity_util import TOL_F32, dev, floored_relerr
from structured_sparse_state_b200.layer import PDSSMLayer, pdssm

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("N,K,D,chunk", [(64, 16, 128, 128), (32, 8, 64, 64), (12, 4, 16, 20)])
def test_function_against_the_oracle(N, K, D, chunk):
    rng = np.random.default_rng(N + K)
    B, H, L = 2, 3, 400
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    W = (rng.standard_normal((H, K, D)) / math.sqrt(D)).astype(np.float32)
    A = rng.standard_normal((K, N, N)).astype(np.float32)
    d = rng.uniform(0.5, 1, (B, H, L, N)).astype(np.float32)
    b = rng.standard_normal((B, H, L, N)).astype(np.float32)
    c = rng.standard_normal((B, H, L, N)).astype(np.float32)
    h0 = rng.standard_normal((B, H, N)).astype(np.float32)
    g_y = rng.standard_normal((B, H, L)).astype(np.float32)
    t = {n: dev(x).requires_grad_() for n, x in dict(W=W, A=A, d=d, b=b, c=c, h0=h0).items()}
    tu = dev(u).requires_grad_()
    y, hl = pdssm(tu, t["W"], t["A"], t["d"], t["b"], t["c"], t["h0"], chunk, 1.3, 0.7)
    (y * dev(g_y)).sum().backward()
    pi = oracle.dict_hardmax(A)
    k = oracle.select(u, W)
    yr, hlr = oracle.scan_fwd(pi, k, d, b, c, h0)
    assert floored_relerr(y.detach().cpu().numpy(), yr) <= TOL_F32
    assert floored_relerr(hl.detach().cpu().numpy(), hlr) <= TOL_F32
    gb, gd, gc, gh0 = oracle.scan_bwd(pi, k, d, b, c, h0, g_y)
    for name, r in (("b", gb), ("d", gd), ("c", gc), ("h0", gh0)):
        assert floored_relerr(t[name].grad.cpu().numpy(), r) <= TOL_F32, name
    gl, gW, gA = oracle.surrogate_grad(u, W, A, 1.3, 0.7, d, b, c, h0, g_y)
    assert floored_relerr(t["W"].grad.cpu().numpy(), gW) <= TOL_F32
    assert floored_relerr(t["A"].grad.cpu().numpy(), gA) <= TOL_F32
    gu = np.einsum("bhlk,hkd->bld", gl, W.astype(np.float64))
    assert floored_relerr(tu.grad.cpu().numpy(), gu) <= TOL_F32


@pytest.mark.parametrize("state_dtype", [torch.float32, torch.bfloat16])
def test_layer_trains_end_to_end(state_dtype):
    torch.manual_seed(0)
    layer = PDSSMLayer(d_model=96, n_heads=4, n_state=32, n_dict=8, d_select=64, chunk=64,
                       state_dtype=state_dtype, device="cuda")
    x = torch.randn(2, 300, 96, device="cuda")
    target = torch.randn(2, 300, 96, device="cuda")
    opt = torch.optim.Adam(layer.parameters(), lr=1e-3)
    losses = []
    for _ in range(5):
        opt.zero_grad()
        loss = torch.nn.functional.mse_loss(layer(x), target)
        loss.backward()
        for name, prm in layer.named_parameters():
            assert prm.grad is not None and torch.isfinite(prm.grad).all(), name
        opt.step()
        losses.append(float(loss))
    assert all(math.isfinite(v) for v in losses)
    assert losses[-1] < losses[0]
