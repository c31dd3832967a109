"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- dense brute force, exact automaton runs (Proposition 1),
closed forms, invariants, exact rational arithmetic and finite differences.

Page references name the page and the section they come from:
  * "Flash PD-SSM technical summary" (gist.science), Methodology §1 hard
    selection / one-hot column selector, §3 three-phase kernel, Main
    contributions (Proposition 1), Experimental results (FSA tasks).
  * "Breaking the Memory Wall" (PGF), abstract: exact derivatives, stiff
    regimes, impulse response.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import pdssm_inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers written independently of the oracle's C code
# ----------------------------------------------------------------------------
def dense_P(pi_row):
    """The one-hot column selector: P[pi(j), j] = 1 (Methodology §1)."""
    N = len(pi_row)
    P = np.zeros((N, N))
    P[pi_row, np.arange(N)] = 1.0
    return P


def dense_forward(pi, k, d, b, c, h0):
    """h_t = P_{k_t} diag(d_t) h_{t-1} + b_t with dense matrices, fp64."""
    B, H, L, N = d.shape
    y = np.zeros((B, H, L))
    hl = np.zeros((B, H, N))
    for bb in range(B):
        for hh in range(H):
            dic = pi if pi.ndim == 2 else pi[hh]
            h = np.zeros(N) if h0 is None else h0[bb, hh].astype(np.float64)
            for t in range(L):
                M = dense_P(dic[k[bb, hh, t]]) @ np.diag(d[bb, hh, t].astype(np.float64))
                h = M @ h + b[bb, hh, t]
                y[bb, hh, t] = c[bb, hh, t] @ h
            hl[bb, hh] = h
    return y, hl


def small_case(seed, B=2, H=3, L=40, N=7, K=5, per_head=False, perms=False):
    rng = np.random.default_rng(seed)
    shape = (H, K, N) if per_head else (K, N)
    if perms:
        pi = np.stack([rng.permutation(N) for _ in range(int(np.prod(shape[:-1])))]
                      ).reshape(shape).astype(np.int32)
    else:
        pi = rng.integers(0, N, size=shape).astype(np.int32)
    k = rng.integers(0, K, size=(B, H, L)).astype(np.int32)
    d = rng.uniform(0.3, 1.2, size=(B, H, L, N))
    b = rng.standard_normal((B, H, L, N))
    c = rng.standard_normal((B, H, L, N))
    h0 = rng.standard_normal((B, H, N))
    return pi, k, d, b, c, h0


def relerr(a, r):
    a = np.asarray(a, np.float64)
    r = np.asarray(r, np.float64)
    scale = max(np.sqrt(np.mean(r * r)) if r.size else 0.0, 1e-300)
    return float(np.max(np.abs(a - r) / np.maximum(np.abs(r), scale))) if r.size else 0.0


# ----------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("N", [1, 2, 5, 8])
def test_forward_matches_dense_bruteforce(per_head, N):
    pi, k, d, b, c, h0 = small_case(10 + N, N=N, per_head=per_head)
    y, hl = oracle.scan_fwd(pi, k, d, b, c, h0)
    y_ref, hl_ref = dense_forward(pi, k, d, b, c, h0)
    assert relerr(y, y_ref) < 1e-12
    assert relerr(hl, hl_ref) < 1e-12


def _read_fixture(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, vals = line.split(":", 1)
            rows[key.strip()] = [int(v) for v in vals.split()]
    return rows


def _dfa_run(delta, accept, q0, symbols):
    """Emulate a DFA with one PD layer: h0 = e_q0, d = 1, b = 0, c = accept
    indicator, pi_sigma(q) = delta(q, sigma)  (Proposition 1)."""
    N = len(accept)
    L = len(symbols)
    pi = np.array([[delta[q][s] for q in range(N)] for s in range(len(delta[0]))],
                  dtype=np.int32)
    k = np.array(symbols, dtype=np.int32).reshape(1, 1, L)
    d = np.ones((1, 1, L, N))
    b = np.zeros((1, 1, L, N))
    c = np.tile(np.array(accept, dtype=np.float64), (1, 1, L, 1))
    h0 = np.zeros((1, 1, N))
    h0[0, 0, q0] = 1.0
    y, hl = oracle.scan_fwd(pi, k, d, b, c, h0)
    return y[0, 0], hl[0, 0]


@pytest.mark.parametrize("fixture,delta,accept", [
    ("dfa_parity.txt", [[0, 1], [1, 0]], [0, 1]),
    ("dfa_mod3.txt", [[0, 1], [1, 2], [2, 0]], [1, 0, 0]),
])
def test_dfa_golden_runs(fixture, delta, accept):
    fx = _read_fixture(fixture)
    y, _ = _dfa_run(delta, accept, 0, fx["symbols"])
    assert y.tolist() == [float(a) for a in fx["accept"]]


def test_dfa_random_non_injective_matches_textbook_simulation():
    rng = np.random.default_rng(7)
    for trial in range(20):
        N = int(rng.integers(2, 12))
        S = int(rng.integers(2, 6))
        delta = rng.integers(0, N, size=(N, S)).tolist()
        accept = rng.integers(0, 2, size=N).tolist()
        symbols = rng.integers(0, S, size=60).tolist()
        q = q0 = int(rng.integers(0, N))
        expect = []
        states = []
        for s in symbols:                     # textbook DFA simulation
            q = delta[q][s]
            states.append(q)
            expect.append(float(accept[q]))
        y, hl = _dfa_run(delta, accept, q0, symbols)
        assert y.tolist() == expect
        one_hot = np.zeros(N)
        one_hot[states[-1]] = 1.0
        assert hl.tolist() == one_hot.tolist()


def test_identity_maps_reduce_to_diagonal_scan_closed_form():
    rng = np.random.default_rng(3)
    B, H, L, N, K = 1, 2, 30, 6, 3
    pi = np.tile(np.arange(N, dtype=np.int32), (K, 1))
    k = rng.integers(0, K, size=(B, H, L)).astype(np.int32)
    d = rng.uniform(0.2, 1.5, size=(B, H, L, N))
    b = rng.standard_normal((B, H, L, N))
    c = rng.standard_normal((B, H, L, N))
    h0 = rng.standard_normal((B, H, N))
    y, hl = oracle.scan_fwd(pi, k, d, b, c, h0)
    for hh in range(H):
        for t in range(L):
            h = np.empty(N)
            for i in range(N):
                acc = h0[0, hh, i]
                for s in range(t + 1):
                    acc *= d[0, hh, s, i]
                for s in range(t + 1):
                    w = b[0, hh, s, i]
                    for r in range(s + 1, t + 1):
                        w *= d[0, hh, r, i]
                    acc += w
                h[i] = acc
            assert abs(y[0, hh, t] - c[0, hh, t] @ h) <= 1e-12 * (1 + abs(y[0, hh, t]))
        assert relerr(hl[0, hh], h) < 1e-12


def test_mass_invariant_any_maps_with_scalar_decay():
    """Every column of P sums to one, so with d_t[j] = a_t for all j:
    sum_i h_t[i] = a_t * sum_j h_{t-1}[j] + sum_i b_t[i]."""
    rng = np.random.default_rng(4)
    B, H, L, N, K = 2, 2, 50, 9, 4
    pi = rng.integers(0, N, size=(K, N)).astype(np.int32)
    k = rng.integers(0, K, size=(B, H, L)).astype(np.int32)
    a = rng.uniform(0.5, 1.0, size=(B, H, L))
    d = np.repeat(a[..., None], N, axis=-1)
    b = rng.standard_normal((B, H, L, N))
    c = np.ones((B, H, L, N))
    h0 = rng.standard_normal((B, H, N))
    y, hl = oracle.scan_fwd(pi, k, d, b, c, h0)
    for bb in range(B):
        for hh in range(H):
            m = h0[bb, hh].sum()
            for t in range(L):
                m = a[bb, hh, t] * m + b[bb, hh, t].sum()
                assert abs(y[bb, hh, t] - m) < 1e-11 * (1 + abs(m))


def test_permutations_with_unit_decay_move_mass_bit_exactly():
    rng = np.random.default_rng(5)
    B, H, L, N, K = 1, 3, 64, 16, 6
    pi = np.stack([rng.permutation(N) for _ in range(K)]).astype(np.int32)
    k = rng.integers(0, K, size=(B, H, L)).astype(np.int32)
    d = np.ones((B, H, L, N))
    b = np.zeros((B, H, L, N))
    c = np.ones((B, H, L, N))
    h0 = rng.standard_normal((B, H, N))
    _, hl = oracle.scan_fwd(pi, k, d, b, c, h0)
    for hh in range(H):
        pos = np.arange(N)
        for t in range(L):
            pos = pi[k[0, hh, t]][pos]
        expect = np.empty(N)
        expect[pos] = h0[0, hh]
        assert (hl[0, hh] == expect).all()
        assert sorted(hl[0, hh].tolist()) == sorted(h0[0, hh].tolist())


def test_impulse_response_closed_form_stiff():
    """b_0 = e_0, h0 = 0: the mass follows one path q_t = pi_{k_t}(q_{t-1}),
    so y_t = c_t[q_t] * prod_{s=1..t} d_s[q_{s-1}] (PGF abstract: impulse
    response; log-uniform d down to 1e-4 gives the stiff regime)."""
    cfg = gen.workload(3, H=4, L=3000)
    inp = gen.generate(cfg)
    y, _ = oracle.scan_fwd(inp.pi, inp.k, inp.d, inp.b, inp.c, None)
    for hh in range(4):
        q = 0
        w = 1.0
        for t in range(cfg["L"]):
            if t > 0:                     # step t moves the mass, then scales it
                w *= float(inp.d[0, hh, t, q])
                q = int(inp.pi[inp.k[0, hh, t]][q])
            expect = float(inp.c[0, hh, t, q]) * w
            got = y[0, hh, t]
            assert np.isfinite(got)
            if abs(expect) >= 1e-300:
                assert abs(got - expect) <= 1e-13 * abs(expect)
            else:
                assert abs(got) <= 1e-300


# ----------------------------------------------------------------------------
# chunk transfers (phases A-C)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("chunk", [1, 2, 7, 16, 64, 1000])
def test_chunk_transfers_reproduce_sequential_states(chunk):
    pi, k, d, b, c, h0 = small_case(21, B=1, H=2, L=64, N=6, K=4, per_head=True)
    Pi, Dl, v = oracle.chunk_transfers(pi, k, d, b, chunk)
    L = k.shape[-1]
    C = (L + chunk - 1) // chunk
    assert Pi.shape[2] == C
    for hh in range(2):
        Hc = h0[0, hh].copy()
        for cc in range(C):
            s, e = cc * chunk, min(L, (cc + 1) * chunk)
            # the composed map, composed again here step by step
            pos = np.arange(6)
            for t in range(s, e):
                pos = pi[hh][k[0, hh, t]][pos]
            assert (Pi[0, hh, cc] == pos).all()
            Hc = dense_P(Pi[0, hh, cc]) @ np.diag(Dl[0, hh, cc]) @ Hc + v[0, hh, cc]
            _, hl = oracle.scan_fwd(pi, k[:, :, :e], d[:, :, :e], b[:, :, :e],
                                    c[:, :, :e], h0)
            assert relerr(Hc, hl[0, hh]) < 1e-12


def test_chunk_transfer_equals_dense_product_of_steps():
    pi, k, d, b, _, _ = small_case(22, B=1, H=1, L=9, N=5, K=3)
    Pi, Dl, v = oracle.chunk_transfers(pi, k, d, b, 9)
    M = np.eye(5)
    for t in range(9):
        M = dense_P(pi[k[0, 0, t]]) @ np.diag(d[0, 0, t]) @ M
    assert np.allclose(dense_P(Pi[0, 0, 0]) @ np.diag(Dl[0, 0, 0]), M, rtol=1e-13, atol=0)


def test_composition_law_and_associativity():
    """(P2,D2,v2) o (P1,D1,v1) = (P2 o P1, D1 * D2[P1], P_{P2} diag(D2) v1 + v2),
    checked against dense products of chunk transfers of sub-sequences."""
    pi, k, d, b, _, _ = small_case(23, B=1, H=1, L=30, N=6, K=4)

    def transfer(s, e):
        P, D, v = oracle.chunk_transfers(pi, k[:, :, s:e], d[:, :, s:e], b[:, :, s:e], e - s)
        return P[0, 0, 0], D[0, 0, 0], v[0, 0, 0]

    def compose(T2, T1):
        P2, D2, v2 = T2
        P1, D1, v1 = T1
        return P2[P1], D1 * D2[P1], dense_P(P2) @ (D2 * v1) + v2

    A, Bt, Ct = transfer(0, 8), transfer(8, 19), transfer(19, 30)
    whole = transfer(0, 30)
    left = compose(Ct, compose(Bt, A))
    right = compose(compose(Ct, Bt), A)
    for X in (left, right):
        assert (X[0] == whole[0]).all()
        assert relerr(X[1], whole[1]) < 1e-13
        assert relerr(X[2], whole[2]) < 1e-12


# ----------------------------------------------------------------------------
# adjoint (PGF: exact analytical derivatives)
# ----------------------------------------------------------------------------
def _loss(pi, k, d, b, c, h0, g_y, g_hl):
    y, hl = oracle.scan_fwd(pi, k, d, b, c, h0)
    return float((g_y * y).sum() + (g_hl * hl).sum())


@pytest.mark.parametrize("with_ghl", [False, True])
def test_adjoint_matches_central_finite_differences(with_ghl):
    pi, k, d, b, c, h0 = small_case(31, B=1, H=2, L=12, N=5, K=3, per_head=True)
    rng = np.random.default_rng(32)
    g_y = rng.standard_normal(k.shape)
    g_hl = rng.standard_normal(h0.shape) if with_ghl else np.zeros(h0.shape)
    g_b, g_d, g_c, g_h0 = oracle.scan_bwd(pi, k, d, b, c, h0, g_y,
                                          g_hl if with_ghl else None)
    eps = 1e-6
    for name, arr, grad in (("b", b, g_b), ("d", d, g_d), ("c", c, g_c), ("h0", h0, g_h0)):
        fd = np.empty_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = arr[idx]
            arr[idx] = old + eps
            lp = _loss(pi, k, d, b, c, h0, g_y, g_hl)
            arr[idx] = old - eps
            lm = _loss(pi, k, d, b, c, h0, g_y, g_hl)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        scale = np.abs(fd).max()
        assert np.abs(fd - grad).max() <= 1e-6 * scale, name


def test_adjoint_dot_product_identity_larger():
    """<g_y, y(x + delta) - y(x)> = <dl/dx, delta> for the variables the
    output is linear in (b, c, h0), at a size with many steps."""
    pi, k, d, b, c, h0 = small_case(33, B=2, H=2, L=300, N=12, K=6)
    rng = np.random.default_rng(34)
    g_y = rng.standard_normal(k.shape)
    g_b, g_d, g_c, g_h0 = oracle.scan_bwd(pi, k, d, b, c, h0, g_y)
    y0, _ = oracle.scan_fwd(pi, k, d, b, c, h0)
    for name in ("b", "c", "h0"):
        delta = rng.standard_normal({"b": b, "c": c, "h0": h0}[name].shape)
        args = dict(b=b, c=c, h0=h0)
        args[name] = args[name] + delta
        y1, _ = oracle.scan_fwd(pi, k, d, args["b"], args["c"], args["h0"])
        lhs = float((g_y * (y1 - y0)).sum())
        rhs = float(({"b": g_b, "c": g_c, "h0": g_h0}[name] * delta).sum())
        assert abs(lhs - rhs) <= 1e-9 * (abs(lhs) + abs(rhs) + 1)
    delta = rng.standard_normal(d.shape) * 1e-3
    eps = 1e-4
    lp = float((g_y * oracle.scan_fwd(pi, k, d + eps * delta, b, c, h0)[0]).sum())
    lm = float((g_y * oracle.scan_fwd(pi, k, d - eps * delta, b, c, h0)[0]).sum())
    assert abs((lp - lm) / (2 * eps) - float((g_d * delta).sum())) <= 1e-6 * (1 + abs(lp))


def test_adjoint_empty_sequence_passes_hlast_gradient():
    pi = np.zeros((2, 3), dtype=np.int32)
    k = np.zeros((1, 1, 0), dtype=np.int32)
    z = np.zeros((1, 1, 0, 3))
    h0 = np.ones((1, 1, 3))
    g_hl = np.array([[[1.0, 2.0, 3.0]]])
    g_b, g_d, g_c, g_h0 = oracle.scan_bwd(pi, k, z, z, z, h0, np.zeros((1, 1, 0)), g_hl)
    assert g_h0.tolist() == g_hl.tolist()


# ----------------------------------------------------------------------------
# hard selection (Methodology §1)
# ----------------------------------------------------------------------------
def _round_f32(fr: Fraction) -> np.float32:
    """Round an exact rational to the nearest float32, ties to even."""
    f = np.float32(float(fr))
    best = None
    for cand in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        if not np.isfinite(cand):
            continue
        err = abs(Fraction(float(cand)) - fr)
        key = (err, int(np.frombuffer(np.float32(cand).tobytes(), np.uint32)[0]) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return best[1]


def test_select_fma_chain_matches_exact_rational_rounding():
    rng = np.random.default_rng(41)
    B, L, D, H, K = 1, 24, 16, 2, 4
    u = rng.standard_normal((B, L, D)).astype(np.float32)
    W = (rng.standard_normal((H, K, D)) / 4).astype(np.float32)
    k = oracle.select(u, W)
    for t in range(L):
        for h in range(H):
            logits = []
            for kk in range(K):
                acc = np.float32(0.0)
                for q in range(D):
                    acc = _round_f32(Fraction(float(W[h, kk, q])) * Fraction(float(u[0, t, q]))
                                     + Fraction(float(acc)))
                logits.append(acc)
            first = max(range(K), key=lambda i: (logits[i], -i))
            assert k[0, h, t] == first


def test_select_agrees_with_fp64_matmul_away_from_ties():
    cfg = gen.workload(1, B=2, L=300)
    inp = gen.generate(cfg)
    k = oracle.select(inp.u, inp.W)
    logits = np.einsum("bld,hkd->bhlk", inp.u.astype(np.float64), inp.W.astype(np.float64))
    srt = np.sort(logits, axis=-1)
    gap = srt[..., -1] - srt[..., -2]
    clear = gap > 1e-4
    assert clear.mean() > 0.99
    assert (k[clear] == np.argmax(logits, axis=-1)[clear]).all()


def test_select_unit_vector_weights_pick_largest_component_and_first_tie():
    u = np.array([[[0.5, -1.0, 2.0, 2.0], [3.0, 3.0, 3.0, 1.0]]], dtype=np.float32)
    W = np.eye(4, dtype=np.float32)[None]          # logit k = u[k]
    k = oracle.select(u, W)
    assert k[0, 0].tolist() == [2, 0]
