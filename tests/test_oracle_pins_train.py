"""Pins of the oracle's dictionary-from-dense-matrices, soft-selection and
surrogate-gradient functions (CPU only).

Flash PD-SSM technical summary:
  * Methodology §1 -- the original PD-SSM mixes dense dictionary matrices
    with soft weights and sparsifies the mixture by a column hardmax; Flash
    PD-SSM keeps K column-hardmax selectors and picks one per step.
  * Methodology §2 -- straight-through estimator: hard forward, tempered
    softmax in the backward so that gradients reach the selection weights
    and the dictionary matrices.
Each pin checks a property the pages or the mathematics fix, by a route that
does not retype the oracle's code: numpy's argmax, the library exp, dense
matrices, a textbook automaton run, finite differences."""
import math

import numpy as np
import pytest

import oracle


def relerr(a, r):
    a = np.asarray(a, np.float64)
    r = np.asarray(r, np.float64)
    scale = max(float(np.sqrt(np.mean(r * r))), 1e-300)
    return float(np.max(np.abs(a - r) / np.maximum(np.abs(r), scale)))


# ----------------------------------------------------------------------------
# column hardmax
# ----------------------------------------------------------------------------
def test_dict_hardmax_is_numpy_first_argmax_over_rows():
    rng = np.random.default_rng(1)
    A = rng.standard_normal((2, 6, 16, 16)).astype(np.float32)
    A[0, 1, 3, 5] = A[0, 1, 9, 5] = 50.0          # a tie: the first row wins
    pi = oracle.dict_hardmax(A)
    assert pi.shape == (2, 6, 16)
    assert (pi == np.argmax(A, axis=-2)).all()
    assert pi[0, 1, 5] == 3


def test_dict_hardmax_recovers_the_map_of_a_one_hot_column_selector():
    """A column one-hot matrix P[pi(j), j] = 1 (the Flash dictionary's form)
    gives back pi, also with noise below the ones."""
    rng = np.random.default_rng(2)
    for N in (1, 5, 32, 64):
        pi = rng.integers(0, N, size=(4, N))
        A = rng.uniform(-1, 0.9, size=(4, N, N)).astype(np.float32)
        for m in range(4):
            A[m, pi[m], np.arange(N)] = 1.0
        assert (oracle.dict_hardmax(A) == pi).all()


# ----------------------------------------------------------------------------
# the soft selection's exp
# ----------------------------------------------------------------------------
def test_soft_exp_against_the_library_exp():
    x = np.concatenate([np.linspace(-86, 0, 200001), -np.logspace(-8, 1.9, 2000), [0.0]])
    x = x.astype(np.float32)
    e = oracle.soft_exp(x).astype(np.float64)
    r = np.exp(x.astype(np.float64))
    assert np.max(np.abs(e - r) / r) < 2e-7
    assert oracle.soft_exp(np.float32([0.0]))[0] == 1.0
    assert (oracle.soft_exp(np.float32([-86.5, -200.0, -1e30])) == 0).all()
    # monotone on a sorted grid
    xs = np.sort(x)
    assert (np.diff(oracle.soft_exp(xs).astype(np.float64)) >= 0).all()


# ----------------------------------------------------------------------------
# soft-selection maps
# ----------------------------------------------------------------------------
def _soft_case(seed, B=2, H=3, L=20, D=12, K=4, N=8):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((B, L, D)).astype(np.float32)
    W = (rng.standard_normal((H, K, D)) / math.sqrt(D)).astype(np.float32)
    A = rng.standard_normal((K, N, N)).astype(np.float32)
    return u, W, A


def test_soft_maps_of_equal_matrices_are_their_hardmax():
    """Any convex combination of K copies of one matrix has its column
    hardmax, whatever the weights."""
    u, W, A = _soft_case(3)
    A[:] = A[0]
    maps = oracle.soft_maps(u, W, A, 1.0)
    want = oracle.dict_hardmax(A[0])
    assert (maps == want).all()


def test_soft_maps_in_the_hard_limit_are_the_flash_selection():
    """With a very small temperature the weights are one-hot on the argmax
    (the other exponentials underflow), so the mixture is the selected
    matrix itself and its hardmax is the Flash dictionary entry."""
    u, W, A = _soft_case(4, K=6, N=16)
    maps = oracle.soft_maps(u, W, A, 1e6)
    k = oracle.select(u, W)
    pi = oracle.dict_hardmax(A)
    lg = np.einsum("hkd,bld->bhlk", W.astype(np.float64), u.astype(np.float64))
    top2 = np.sort(lg, axis=-1)[..., -2:]
    clear = (top2[..., 1] - top2[..., 0]) > 1e-3
    assert clear.mean() > 0.9
    want = pi[k]                                       # [B, H, L, N]
    assert (maps[clear] == want[clear]).all()


def test_soft_maps_follow_a_row_permutation_of_the_matrices():
    """Relabelling the rows of every A_k by sigma relabels every map value by
    sigma (catches a row/column mix-up)."""
    u, W, A = _soft_case(5)
    sigma = np.random.default_rng(9).permutation(A.shape[-1])
    A2 = np.empty_like(A)
    A2[:, sigma, :] = A
    m1 = oracle.soft_maps(u, W, A, 0.7)
    m2 = oracle.soft_maps(u, W, A2, 0.7)
    assert (m2 == sigma[m1]).all()


def test_soft_maps_mix_matrices_when_weights_are_balanced():
    """Two matrices whose hardmax rows differ and equal weights (identical
    weight rows): each column's winner is the row of the larger summed entry,
    computed here from the dense sum."""
    N, K, D = 6, 2, 4
    rng = np.random.default_rng(6)
    A = rng.uniform(0, 1, (K, N, N)).astype(np.float32)
    W = np.tile(rng.standard_normal((1, 1, D)), (1, K, 1)).astype(np.float32)
    u = rng.standard_normal((1, 5, D)).astype(np.float32)
    maps = oracle.soft_maps(u, W, A, 1.0)
    want = np.argmax(A.astype(np.float64).sum(0), axis=0)
    assert (maps == want).all()


# ----------------------------------------------------------------------------
# forward scan with one map per step
# ----------------------------------------------------------------------------
def test_scan_fwd_maps_matches_dense_matrices():
    rng = np.random.default_rng(7)
    B, H, L, N = 2, 2, 30, 6
    maps = rng.integers(0, N, size=(B, H, L, N)).astype(np.int32)
    d = rng.uniform(0.3, 1.2, (B, H, L, N))
    b = rng.standard_normal((B, H, L, N))
    c = rng.standard_normal((B, H, L, N))
    h0 = rng.standard_normal((B, H, N))
    y, hl = oracle.scan_fwd_maps(maps, d, b, c, h0)
    for bb in range(B):
        for hh in range(H):
            h = h0[bb, hh].copy()
            for t in range(L):
                P = np.zeros((N, N))
                P[maps[bb, hh, t], np.arange(N)] = 1.0
                h = P @ (d[bb, hh, t] * h) + b[bb, hh, t]
                assert abs(y[bb, hh, t] - c[bb, hh, t] @ h) <= 1e-12 * (1 + abs(y[bb, hh, t]))
            assert np.allclose(hl[bb, hh], h, rtol=1e-12, atol=1e-12)


def test_scan_fwd_maps_runs_a_time_varying_automaton():
    """Per-step transition functions (an input-dependent automaton): with
    h0 = e_q0, d = 1, b = 0 and c the accept indicator, y_t is 1 exactly when
    the textbook run is in an accepting state."""
    rng = np.random.default_rng(8)
    N, L = 5, 200
    maps = rng.integers(0, N, size=(1, 1, L, N)).astype(np.int32)
    accept = rng.integers(0, 2, N).astype(np.float64)
    q = 2
    want = []
    for t in range(L):
        q = maps[0, 0, t, q]
        want.append(accept[q])
    h0 = np.zeros((1, 1, N))
    h0[0, 0, 2] = 1.0
    y, _ = oracle.scan_fwd_maps(maps, np.ones((1, 1, L, N)), np.zeros((1, 1, L, N)),
                                np.tile(accept, (1, 1, L, 1)), h0)
    assert (y[0, 0] == np.array(want)).all()


def test_scan_fwd_maps_equals_dictionary_scan_on_dictionary_maps():
    rng = np.random.default_rng(10)
    B, H, L, N, K = 2, 2, 50, 7, 3
    pi = rng.integers(0, N, size=(K, N)).astype(np.int32)
    k = rng.integers(0, K, size=(B, H, L)).astype(np.int32)
    d = rng.uniform(0.5, 1, (B, H, L, N))
    b = rng.standard_normal((B, H, L, N))
    c = rng.standard_normal((B, H, L, N))
    y1, h1 = oracle.scan_fwd_maps(pi[k], d, b, c)
    y2, h2 = oracle.scan_fwd(pi, k, d, b, c)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


# ----------------------------------------------------------------------------
# straight-through surrogate gradients
# ----------------------------------------------------------------------------
def _train_case(seed, B=2, H=2, L=12, N=5, K=3, D=6, per_head=False):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((B, L, D)).astype(np.float32)
    W = (rng.standard_normal((H, K, D)) / math.sqrt(D)).astype(np.float32)
    A = rng.standard_normal(((H,) if per_head else ()) + (K, N, N)).astype(np.float32)
    d = rng.uniform(0.5, 1.0, (B, H, L, N))
    b = rng.standard_normal((B, H, L, N))
    c = rng.standard_normal((B, H, L, N))
    h0 = rng.standard_normal((B, H, N))
    g_y = rng.standard_normal((B, H, L))
    return u, W, A, d, b, c, h0, g_y


def _hard_trajectory(u, W, A, d, b, c, h0, g_y):
    """lambda_t (the adjoint of the hard model) and z_t = d_t h_{t-1}."""
    pi = oracle.dict_hardmax(A)
    k = oracle.select(u, W)
    lam = oracle.scan_bwd(pi, k, d, b, c, h0, g_y)[0]
    B, H, L, N = d.shape
    hprev = np.empty((B, H, L, N))
    hprev[:, :, 0] = h0
    for t in range(1, L):
        hprev[:, :, t] = oracle.scan_fwd(pi, k[:, :, :t], d[:, :, :t], b[:, :, :t],
                                         c[:, :, :t], h0)[1]
    return lam, d * hprev


def _softmax(x, axis):
    x = x - x.max(axis=axis, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=axis, keepdims=True)


def _sel_loss(u, W, pi, inv_s, lam, z):
    """G_sel(W) = sum_t lambda_t^T (sum_k s_{t,k} P_k) z_t, with dense P_k."""
    lg = np.einsum("hkd,bld->bhlk", W, u.astype(np.float64))
    s = _softmax(lg * inv_s, axis=-1)
    N = pi.shape[-1]
    P = np.zeros(pi.shape[:-1] + (N, N))
    np.put_along_axis(P, pi[..., None, :], 1.0, axis=-2)
    if P.ndim == 3:
        return float(np.einsum("bhlk,bhli,kij,bhlj->", s, lam, P, z))
    return float(np.einsum("bhlk,bhli,hkij,bhlj->", s, lam, P, z))


def _dict_loss(A, k, inv_a, lam, z):
    """G_dict(A) = sum_t lambda_t^T Q_{k_t} z_t, Q the column softmaxes."""
    Q = _softmax(A * inv_a, axis=-2)
    B, H, L = k.shape
    total = 0.0
    for bb in range(B):
        for hh in range(H):
            for t in range(L):
                Qk = Q[k[bb, hh, t]] if Q.ndim == 3 else Q[hh, k[bb, hh, t]]
                total += lam[bb, hh, t] @ Qk @ z[bb, hh, t]
    return total


@pytest.mark.parametrize("per_head", [False, True])
def test_surrogate_gradients_match_finite_differences_of_the_linearised_losses(per_head):
    u, W, A, d, b, c, h0, g_y = _train_case(11, per_head=per_head)
    inv_s, inv_a = 1.7, 2.3
    g_l, g_W, g_A = oracle.surrogate_grad(u, W, A, inv_s, inv_a, d, b, c, h0, g_y)
    lam, z = _hard_trajectory(u, W, A, d, b, c, h0, g_y)
    pi = oracle.dict_hardmax(A)
    k = oracle.select(u, W)
    W64, A64 = W.astype(np.float64), A.astype(np.float64)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for _ in range(12):
        idx = tuple(int(rng.integers(0, n)) for n in W.shape)
        Wp, Wm = W64.copy(), W64.copy()
        Wp[idx] += eps
        Wm[idx] -= eps
        fd = (_sel_loss(u, Wp, pi, inv_s, lam, z) - _sel_loss(u, Wm, pi, inv_s, lam, z)) / (2 * eps)
        assert abs(fd - g_W[idx]) <= 1e-5 * max(1.0, abs(fd)), (idx, fd, g_W[idx])
    for _ in range(12):
        idx = tuple(int(rng.integers(0, n)) for n in A.shape)
        Ap, Am = A64.copy(), A64.copy()
        Ap[idx] += eps
        Am[idx] -= eps
        fd = (_dict_loss(Ap, k, inv_a, lam, z) - _dict_loss(Am, k, inv_a, lam, z)) / (2 * eps)
        assert abs(fd - g_A[idx]) <= 1e-5 * max(1.0, abs(fd)), (idx, fd, g_A[idx])
    # the logit gradients are the same derivative taken at the logits
    lg = np.einsum("hkd,bld->bhlk", W64, u.astype(np.float64))
    for _ in range(6):
        bb, hh, t, kk = (int(rng.integers(0, n)) for n in g_l.shape)
        P = np.zeros(pi.shape[:-1] + (pi.shape[-1],) * 2)
        np.put_along_axis(P, pi[..., None, :], 1.0, axis=-2)
        Pk = P if P.ndim == 3 else P[hh]

        def at(delta):
            x = lg[bb, hh, t].copy()
            x[kk] += delta
            s = _softmax(x * inv_s, axis=-1)
            return float(np.einsum("k,i,kij,j->", s, lam[bb, hh, t], Pk, z[bb, hh, t]))
        fd = (at(eps) - at(-eps)) / (2 * eps)
        assert abs(fd - g_l[bb, hh, t, kk]) <= 1e-5 * max(1.0, abs(fd))


def test_surrogate_logit_gradients_sum_to_zero_and_vanish_for_equal_matrices():
    """softmax is invariant to a common shift of the logits, so each step's
    logit gradients sum to zero; with all A_k equal every selector is the
    same, so the relaxed transition does not depend on the weights at all."""
    u, W, A, d, b, c, h0, g_y = _train_case(12)
    g_l, g_W, g_A = oracle.surrogate_grad(u, W, A, 1.3, 1.0, d, b, c, h0, g_y)
    assert np.max(np.abs(g_l.sum(-1))) <= 1e-12 * max(1.0, np.max(np.abs(g_l)))
    assert np.max(np.abs(g_l)) > 1e-3
    A[:] = A[0]
    g_l, g_W, _ = oracle.surrogate_grad(u, W, A, 1.3, 1.0, d, b, c, h0, g_y)
    assert np.max(np.abs(g_l)) <= 1e-12 and np.max(np.abs(g_W)) <= 1e-12


def test_surrogate_dictionary_gradient_columns_sum_to_zero():
    """Each column of Q_k is a softmax over rows, so the gradient of its
    logits sums to zero down every column."""
    u, W, A, d, b, c, h0, g_y = _train_case(13)
    _, _, g_A = oracle.surrogate_grad(u, W, A, 1.0, 0.8, d, b, c, h0, g_y)
    assert np.max(np.abs(g_A.sum(-2))) <= 1e-12 * max(1.0, np.max(np.abs(g_A)))
