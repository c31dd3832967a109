"""Multi-head Flash PD-SSM layer over the C ABI.

Flash PD-SSM technical summary, Methodology §4: the SSM sits in a standard
pre-norm architecture as a multi-head layer, and the heads share the dense
dictionary matrices (which amortises their parameters); §1: the dictionary
is the column hardmax of those matrices and each step selects one entry by
the argmax of K linear scores; §2: the backward replaces the discrete
choices by tempered softmaxes (straight-through).

``PDSSMFunction`` is the differentiable core, every step in the library's
kernels: the dictionary (pdssm_dict_hardmax), the selection (pdssm_select),
the single-pass forward (pdssm_scan_fwd), the exact adjoint for d, b, c and
h0 (pdssm_scan_bwd) and the surrogate gradients for W_sel and the dictionary
matrices (pdssm_surrogate_bwd).  The one product outside the library is the
gradient with respect to u, g_u = g_logits . W_sel, a plain GEMM.

``PDSSMLayer`` wraps it in a pre-norm residual block with its projections
(RMS norm, linear maps for u, d, b, c and the output), which are ordinary
library operations.
"""
from __future__ import annotations

import torch

from . import (pdssm_dict_hardmax, pdssm_scan_bwd, pdssm_scan_fwd, pdssm_select,
               pdssm_surrogate_bwd)


class PDSSMFunction(torch.autograd.Function):
    """(u, W_sel, A, d, b, c, h0) -> (y, h_last) of the hard model."""

    @staticmethod
    def forward(ctx, u, W_sel, A, d, b, c, h0, chunk, inv_tau_s, inv_tau_a):
        pi = pdssm_dict_hardmax(A)
        k = pdssm_select(u, W_sel)
        y, h_last, ws = pdssm_scan_fwd(pi, k, d, b, c, h0, chunk=chunk, for_bwd=True)
        ctx.save_for_backward(u, W_sel, A, d, b, c, h0, pi, k, ws)
        ctx.chunk, ctx.inv_tau_s, ctx.inv_tau_a = chunk, inv_tau_s, inv_tau_a
        return y, h_last

    @staticmethod
    def backward(ctx, g_y, g_hlast):
        u, W_sel, A, d, b, c, h0, pi, k, ws = ctx.saved_tensors
        g_y = torch.zeros_like(k, dtype=torch.float32) if g_y is None else g_y.float().contiguous()
        g_hl = None if g_hlast is None else g_hlast.float().contiguous()
        g_b, g_d, g_c, g_h0 = pdssm_scan_bwd(pi, k, d, b, c, h0, g_y, ws, chunk=ctx.chunk,
                                             g_hlast=g_hl)
        g_l, g_W, g_A = pdssm_surrogate_bwd(u, W_sel, A, pi, k, d, b, h0, g_b, ws, ctx.chunk,
                                            ctx.inv_tau_s, ctx.inv_tau_a)
        # dl/du[b, t, :] = sum_{h, k} g_logits[b, h, t, k] W_sel[h, k, :]
        B, H, L, K = g_l.shape
        g_u = torch.matmul(g_l.permute(0, 2, 1, 3).reshape(B, L, H * K),
                           W_sel.reshape(H * K, -1))
        return (g_u.to(u.dtype), g_W, g_A, g_d.to(d.dtype), g_b.to(b.dtype), g_c.to(c.dtype),
                g_h0 if h0 is not None else None, None, None, None)


def pdssm(u, W_sel, A, d, b, c, h0=None, chunk=128, inv_tau_s=1.0, inv_tau_a=1.0):
    """Differentiable hard-selection PD-SSM: returns (y [B, H, L], h_last)."""
    return PDSSMFunction.apply(u, W_sel, A, d, b, c, h0, chunk, inv_tau_s, inv_tau_a)


class PDSSMLayer(torch.nn.Module):
    """Pre-norm residual multi-head PD-SSM block:
        x -> x + W_out y,  y = PD-SSM(u, d, b, c) of RMSNorm(x),
    u = W_u x_n (selection input), d = sigmoid(W_d x_n), b = W_b x_n,
    c = W_c x_n per head, a dictionary of K dense N x N matrices shared by
    the heads.  Inputs [B, L, d_model]; d, b, c in `state_dtype`."""

    def __init__(self, d_model, n_heads, n_state, n_dict, d_select=None, chunk=128,
                 inv_tau_s=1.0, inv_tau_a=1.0, state_dtype=torch.float32, device=None):
        super().__init__()
        d_select = d_select or d_model
        self.H, self.N, self.K, self.D = n_heads, n_state, n_dict, d_select
        self.chunk, self.inv_tau_s, self.inv_tau_a = chunk, inv_tau_s, inv_tau_a
        self.state_dtype = state_dtype
        f = dict(device=device, dtype=torch.float32)
        self.norm = torch.nn.RMSNorm(d_model, **f)
        self.proj_u = torch.nn.Linear(d_model, d_select, bias=False, **f)
        self.proj_d = torch.nn.Linear(d_model, n_heads * n_state, **f)
        self.proj_b = torch.nn.Linear(d_model, n_heads * n_state, bias=False, **f)
        self.proj_c = torch.nn.Linear(d_model, n_heads * n_state, bias=False, **f)
        self.W_sel = torch.nn.Parameter(torch.randn(n_heads, n_dict, d_select, **f) /
                                        d_select ** 0.5)
        self.A = torch.nn.Parameter(torch.randn(n_dict, n_state, n_state, **f))
        self.proj_out = torch.nn.Linear(n_heads, d_model, bias=False, **f)
        with torch.no_grad():
            self.proj_d.bias.fill_(2.0)   # decays start near sigmoid(2)

    def _heads(self, t, B, L):
        return t.view(B, L, self.H, self.N).permute(0, 2, 1, 3).contiguous().to(self.state_dtype)

    def forward(self, x):
        B, L, _ = x.shape
        xn = self.norm(x)
        u = self.proj_u(xn)
        if self.state_dtype == torch.bfloat16:
            u = u.to(torch.bfloat16)
        d = self._heads(torch.sigmoid(self.proj_d(xn)), B, L)
        b = self._heads(self.proj_b(xn), B, L)
        c = self._heads(self.proj_c(xn), B, L)
        y, _ = pdssm(u.contiguous(), self.W_sel, self.A, d, b, c, None, self.chunk,
                     self.inv_tau_s, self.inv_tau_a)
        return x + self.proj_out(y.permute(0, 2, 1))
