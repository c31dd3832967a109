"""GPU parity: the sm_100a kernels, called through the C ABI, against the CPU
oracle on the same seeded inputs.  Indices (k, composed maps) must match bit
for bit; floats within the floored relative error of 1e-5 (fp32 inputs) or
2e-2 (bf16 inputs)."""
import numpy as np
import pytest
import torch

import oracle
import pdssm_inputs as gen
import structured_sparse_state_b200 as pd
from parity_util import (TOL_F32, dev, floored_relerr, oracle_k, sample_rows, to_device,
                         tol_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def run_fwd(inp, chunk, k=None, for_bwd=False):
    t = to_device(inp)
    kk = k if k is not None else t["k"]
    y, hl, ws = pd.pdssm_scan_fwd(t["pi"], kk, t["d"], t["b"], t["c"], t["h0"], chunk=chunk,
                                  for_bwd=for_bwd)
    assert pd.pdssm_ws_status(ws) == 0
    return t, kk, y, hl, ws


def check_fwd(inp, chunk, k_np=None, single=False):
    t = to_device(inp)
    if k_np is None:
        k_np = oracle_k(inp)
    kk = dev(k_np, torch.int32)
    fwd = pd.pdssm_scan_fwd_single_pass if single else pd.pdssm_scan_fwd
    y, hl, ws = fwd(t["pi"], kk, t["d"], t["b"], t["c"], t["h0"], chunk=chunk)
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws) == 0
    y_ref, hl_ref = oracle.scan_fwd(inp.pi, k_np, inp.d, inp.b, inp.c, inp.h0)
    tol = tol_for(inp)
    ey = floored_relerr(y.cpu().numpy(), y_ref)
    eh = floored_relerr(hl.cpu().numpy(), hl_ref)
    assert ey <= tol, f"y error {ey}"
    assert eh <= tol, f"h_last error {eh}"
    return ey, eh


# ----------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("idx,over", [(0, {}), (1, dict(B=2, L=1500)),
                                      (2, dict(B=1, L=777)), (2, dict(B=2, L=130, K=5))])
def test_select_bit_exact(idx, over):
    inp = gen.generate(gen.workload(idx, **over))
    t = to_device(inp)
    k = pd.pdssm_select(t["u"], t["W"]).cpu().numpy()
    assert (k == oracle.select(inp.u, inp.W)).all()


@pytest.mark.parametrize("H,K,D", [(16, 16, 128), (2, 8, 64), (1, 4, 16), (4, 32, 32),
                                   (3, 2, 48), (4, 16, 192), (2, 8, 256), (5, 1, 64)])
def test_select_tensor_core_shapes_bit_exact(H, K, D):
    """bf16 u with K a power of two takes the tcgen05 path (certified
    argmax, exact fma-chain recompute near ties); D a multiple of 64 uses
    the 128-byte swizzled operands (1 to 4 atoms), other D the unswizzled
    ones; K = 1 has a single candidate per head."""
    rng = np.random.default_rng(H * 1000 + K * 10 + D)
    B, L = 2, 333
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    W = (rng.standard_normal((H, K, D)) / np.sqrt(D)).astype(np.float32)
    k = pd.pdssm_select(dev(u, bf16=True), dev(W)).cpu().numpy()
    assert (k == oracle.select(u, W)).all()


@pytest.mark.parametrize("bf16", [True, False])
def test_select_largest_sizes(bf16):
    """K = 32 and D_in = 256, the boundary's limits, with H*K = 256 scores per
    row (the tensor-core kernel's operands would not fit its shared memory,
    so the fma-chain kernel decides); bit-exact for bf16 and fp32 u."""
    rng = np.random.default_rng(256)
    H, K, D, B, L = 8, 32, 256, 2, 300
    u = rng.standard_normal((B, L, D)).astype(np.float32)
    if bf16:
        u = gen.round_bf16(u)
    W = (rng.standard_normal((H, K, D)) / np.sqrt(D)).astype(np.float32)
    k = pd.pdssm_select(dev(u, bf16=bf16), dev(W)).cpu().numpy()
    assert (k == oracle.select(u, W)).all()


def test_select_near_ties_take_the_exact_path():
    """Rows of W that differ by ~1e-6 make most top-2 gaps smaller than the
    certification bound, so the exact fma chains decide."""
    rng = np.random.default_rng(77)
    H, K, D, B, L = 4, 16, 128, 1, 512
    base = (rng.standard_normal((H, 1, D)) / np.sqrt(D)).astype(np.float32)
    W = (base + 1e-6 * rng.standard_normal((H, K, D))).astype(np.float32)
    W[:, 5] = W[:, 3]                        # exact duplicates: first index wins
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    k = pd.pdssm_select(dev(u, bf16=True), dev(W)).cpu().numpy()
    kr = oracle.select(u, W)
    assert (k == kr).all()
    assert not (kr == 5).any() or (kr == 3).any()


def test_select_full_size_tensor_core_equals_fma_kernel():
    """The full bf16 selection workload: the tensor-core route and the plain
    fma-chain route agree on every index, and a sample of rows matches the
    oracle."""
    inp = gen.generate(gen.workload(2))
    u = dev(inp.u, bf16=True)
    W = dev(inp.W)
    k_tc = pd.pdssm_select(u, W, method="tensor_core").cpu().numpy()
    k_fma = pd.pdssm_select(u, W, method="fma").cpu().numpy()
    assert (k_tc == k_fma).all()
    assert (pd.pdssm_select(u, W).cpu().numpy() == k_tc).all()
    rows = [0, 1, 7, 4095, 9999, 16383]
    for b in (0, 5):
        kr = oracle.select(inp.u[b:b + 1, rows], inp.W)
        assert (k_tc[b][:, rows] == kr[0]).all()


def _exact_logits(u, W):
    """Exact (fp64) sums u . W for bf16-valued u and fp32 W: every product is
    exact in fp64 and D <= 256 sums of them lose far less than the bounds
    checked here."""
    B, L, D = u.shape
    H, K, _ = W.shape
    return u.reshape(B * L, D).astype(np.float64) @ W.reshape(H * K, D).astype(np.float64).T


TC_ACC_BOUND = lambda D: D * 2.0 ** -21 + 2.0 ** -16   # noqa: E731


@pytest.mark.parametrize("H,K,D", [(16, 16, 128), (4, 8, 64), (2, 32, 256), (8, 4, 48)])
def test_select_tensor_core_logits_within_certified_bound(H, K, D):
    """The certification assumes |tensor-core logit - exact sum| <=
    (D 2^-21 + 2^-16) * ||u|| * max_k ||W_hk||.  Check it on raw logits
    read through the test hook, against exact sums."""
    rng = np.random.default_rng(4242 + D)
    B, L = 2, 1000
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    u[0, :10] *= 1e3                       # a few large rows
    u[1, :10] *= 1e-3                      # and a few small ones
    u = gen.round_bf16(u)
    W = (rng.standard_normal((H, K, D)) / np.sqrt(D)).astype(np.float32)
    k, lg, sc = pd.pdssm_select_tc_logits(dev(u, bf16=True), dev(W))
    lg = lg.cpu().numpy().astype(np.float64)
    sc = np.repeat(sc.cpu().numpy().astype(np.float64), K, axis=1)
    exact = _exact_logits(u, W)
    # the scale is ||u|| max ||W_hk||, rounded up
    un = np.sqrt((u.reshape(B * L, D).astype(np.float64) ** 2).sum(1))
    wn = np.sqrt((W.astype(np.float64) ** 2).sum(2)).max(1)
    assert (sc >= np.repeat(un[:, None] * wn[None, :], K, axis=1) * (1 - 1e-12)).all()
    ratio = np.abs(lg - exact) / (TC_ACC_BOUND(D) * sc)
    assert ratio.max() <= 1.0, f"tensor-core error {ratio.max():.3f} x the assumed bound"
    assert (k.cpu().numpy() == oracle.select(u, W)).all()


def test_select_gaps_just_above_the_certification_threshold():
    """Rows whose top-2 gap lies in [2.2, 3.8] x eps (eps = the certification
    half-width) are decided by the single-candidate branch; they must still
    match the fma-chain contract bit for bit.  The two leading weights differ
    only in the coefficient of u_0, so the gap is u_0 times it; the other
    candidates sit far below through u_1."""
    H, K, D, B, L = 4, 16, 128, 2, 2048
    rng = np.random.default_rng(909)
    W = (rng.standard_normal((H, 1, D)) / np.sqrt(D)).astype(np.float32).repeat(K, 1)
    W[:, 1, 0] -= 1.0                          # l_0 - l_1 = u_0
    W[:, 2:, 1] -= 0.5                         # l_k = l_0 - 0.5 u_1 for k >= 2
    u = gen.round_bf16(rng.standard_normal((B, L, D)).astype(np.float32))
    u[:, :, 1] = 4.0
    ceps = 1.01 * (D * 2.0 ** -21 + 2.0 ** -16 + D * 2.0 ** -24)
    wn = np.sqrt((W.astype(np.float64) ** 2).sum(2)).max()
    target = rng.uniform(2.4, 3.6, (B, L)) * np.where(rng.random((B, L)) < 0.5, 1.0, -1.0)
    for _ in range(3):                         # u_0 enters ||u|| slightly
        un = np.sqrt((u.astype(np.float64) ** 2).sum(2))
        u[:, :, 0] = target * ceps * un * wn * 1.002
        u = gen.round_bf16(u)
    ud, Wd = dev(u, bf16=True), dev(W)
    k, lg, sc = pd.pdssm_select_tc_logits(ud, Wd)
    kr = oracle.select(u, W)
    assert (k.cpu().numpy() == kr).all()
    assert set(np.unique(kr)) == {0, 1}
    exact = _exact_logits(u, W).reshape(B * L, H, K)
    gap = np.abs(exact[:, :, 0] - exact[:, :, 1])
    eps = ceps * sc.cpu().numpy().astype(np.float64)
    rel = gap / eps
    assert ((rel > 2.0) & (rel < 4.0)).mean() > 0.95
    lgn = lg.cpu().numpy().reshape(B * L, H, K).astype(np.float64)
    thr = lgn.max(2) - 2 * eps
    single = ((lgn >= thr[:, :, None]).sum(2) == 1)
    assert single.sum() >= 0.9 * B * L * H, "most decisions take the certified branch"
    assert (pd.pdssm_select(ud, Wd, method="fma").cpu().numpy() == kr).all()


# ----------------------------------------------------------------------------
# chunk transfers: composed maps bit-exact
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("idx,over,chunk", [
    (0, {}, 32), (1, dict(B=1, L=1000), 64), (2, dict(B=1, H=2, L=600), 128),
    (3, dict(H=2, L=1000), 256), (4, dict(B=1, H=2, L=700), 128), (4, dict(B=1, H=1, L=50), 7)])
def test_chunk_transfers(idx, over, chunk):
    inp = gen.generate(gen.workload(idx, **over))
    k_np = oracle_k(inp)
    t = to_device(inp)
    Pi, Dl, v = pd.pdssm_chunk_transfers(t["pi"], dev(k_np, torch.int32), t["d"], t["b"], chunk)
    Pi_r, Dl_r, v_r = oracle.chunk_transfers(inp.pi, k_np, inp.d, inp.b, chunk)
    assert (Pi.cpu().numpy() == Pi_r).all()
    tol = tol_for(inp)
    assert floored_relerr(Dl.cpu().numpy(), Dl_r) <= tol
    assert floored_relerr(v.cpu().numpy(), v_r) <= tol


# ----------------------------------------------------------------------------
# single-pass forward (N = 32 / 64, aligned rows): look-back and in-CTA scan
# ----------------------------------------------------------------------------
def _prefix_states(inp, k_np, chunk):
    """Oracle state at the end of every chunk: h_last of each prefix."""
    L = inp.d.shape[2]
    out = []
    for e in range(chunk, L + chunk, chunk):
        e = min(e, L)
        _, h = oracle.scan_fwd(inp.pi, k_np[:, :, :e], inp.d[:, :, :e], inp.b[:, :, :e],
                               inp.c[:, :, :e], inp.h0)
        out.append(h)
    return np.stack(out, axis=2)


@pytest.mark.parametrize("kind", ["maps", "perm"])
@pytest.mark.parametrize("N,dtype", [(32, "f32"), (64, "f32"), (32, "bf16"), (64, "bf16")])
def test_single_pass_transfers_and_carries(N, dtype, kind):
    """After the single-pass forward the workspace holds every chunk's
    composed transfer (maps bit-exact against the oracle's step-by-step
    composition) and the carry at every chunk end (the oracle's state)."""
    inp = small(N + len(kind), 2, 3, 1000, N, 6, kind=kind, dtype=dtype)
    chunk = 64
    t = to_device(inp)
    y, hl, ws = pd.pdssm_scan_fwd_single_pass(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"],
                                              chunk=chunk)
    Pi, Dl, v, Hc = pd.pdssm_ws_transfers(ws, 2, 3, 1000, N, 6, chunk)
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws) == 0
    Pi_r, Dl_r, v_r = oracle.chunk_transfers(inp.pi, inp.k, inp.d, inp.b, chunk)
    assert (Pi.cpu().numpy() == Pi_r).all()
    tol = tol_for(inp)
    assert floored_relerr(Dl.cpu().numpy(), Dl_r) <= tol
    assert floored_relerr(v.cpu().numpy(), v_r) <= tol
    assert floored_relerr(Hc.cpu().numpy(), _prefix_states(inp, inp.k, chunk)) <= tol


@pytest.mark.parametrize("chunk", [1, 3, 7, 8, 9, 15, 17, 63, 65, 300])
@pytest.mark.parametrize("N", [32, 64])
def test_single_pass_chunk_sizes(chunk, N):
    """Chunks shorter than the CTA's eight sub-chunks leave warps with empty
    sub-chunks; ragged chunks and tails throughout."""
    check_fwd(small(chunk + N, 1, 3, 777, N, 5), chunk=chunk, single=True)


@pytest.mark.parametrize("N,kind", [(32, "perm"), (64, "maps")])
def test_single_pass_long_look_back(N, kind):
    """One sequence of 60000 steps in chunks of 8: hundreds of chunks of the
    same sequence run at once, so look-backs walk back over whole windows of
    published aggregates."""
    check_fwd(small(5, 1, 1, 60000, N, 8, kind=kind), chunk=8, single=True)


@pytest.mark.parametrize("idx,over", [(2, dict(B=2, H=3, L=1000)), (3, dict(H=4, L=3000)),
                                      (4, dict(B=1, H=3, L=2000))])
def test_single_pass_workloads_reduced(idx, over):
    inp = gen.generate(gen.workload(idx, **over))
    check_fwd(inp, inp.cfg["chunk"], single=True)


def test_single_pass_then_backward():
    """The single-pass forward leaves the workspace the adjoint reads: the
    backward after it matches the oracle."""
    inp = small(9, 2, 2, 700, 64, 6)
    t = to_device(inp)
    y, hl, ws = pd.pdssm_scan_fwd_single_pass(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"],
                                              chunk=64, for_bwd=True)
    g = pd.pdssm_scan_bwd(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"], t["g_y"], ws, chunk=64)
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws) == 0
    ref = oracle.scan_bwd(inp.pi, inp.k, inp.d, inp.b, inp.c, inp.h0, inp.g_y)
    for a, r in zip(g, ref):
        assert floored_relerr(a.cpu().numpy(), r) <= TOL_F32


def test_single_pass_rejects_unsupported_shapes():
    inp = small(1, 1, 1, 50, 24, 3)
    t = to_device(inp)
    with pytest.raises(pd.PdssmError):
        pd.pdssm_scan_fwd_single_pass(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"], chunk=16)


@pytest.mark.parametrize("idx", [2, 3])
def test_single_pass_full_size_equals_three_kernels(idx):
    """Full benchmark sizes: the single-pass forward and the three-kernel
    forward agree within the workload's tolerance (and bitwise-equal
    integer transfers), and each is deterministic."""
    cfg = gen.workload(idx)
    inp = gen.generate(cfg)
    t = to_device(inp)
    k = t["k"] if t["k"] is not None else pd.pdssm_select(t["u"], t["W"])
    y3, h3, ws3 = pd.pdssm_scan_fwd(t["pi"], k, t["d"], t["b"], t["c"], t["h0"], chunk=cfg["chunk"])
    y1, h1, ws1 = pd.pdssm_scan_fwd_single_pass(t["pi"], k, t["d"], t["b"], t["c"], t["h0"],
                                                chunk=cfg["chunk"])
    y1b, h1b, _ = pd.pdssm_scan_fwd_single_pass(t["pi"], k, t["d"], t["b"], t["c"], t["h0"],
                                                chunk=cfg["chunk"])
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws1) == 0
    assert torch.equal(y1, y1b) and torch.equal(h1, h1b)
    tol = tol_for(inp)
    assert floored_relerr(y1.cpu().numpy(), y3.cpu().numpy()) <= tol
    assert floored_relerr(h1.cpu().numpy(), h3.cpu().numpy()) <= tol
    B, H, L, N = inp.d.shape
    P1 = pd.pdssm_ws_transfers(ws1, B, H, L, N, cfg["K"], cfg["chunk"])[0]
    P3 = pd.pdssm_ws_transfers(ws3, B, H, L, N, cfg["K"], cfg["chunk"])[0]
    assert torch.equal(P1, P3)


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_waits_time_out_and_report(which):
    """A wait that nothing completes (a look-back flag no chunk publishes; an
    mbarrier no copy completes) gives up after its cap and the host reads
    PDSSM_ERR_TIMEOUT from the status word; the context stays usable."""
    assert pd.pdssm_wait_selftest(which, 1_000_000) == 5
    inp = small(3, 1, 1, 100, 32, 3)
    check_fwd(inp, chunk=16)


# ----------------------------------------------------------------------------
# forward, reduced copies of the five workloads (several tiles, ragged tails)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("idx,over", [
    (0, {}),
    (1, {}),
    (2, dict(B=2, H=3, L=1000)),
    (3, dict(H=4, L=3000)),
    (4, dict(B=1, H=3, L=2000)),
])
def test_forward_workloads_reduced(idx, over):
    cfg = gen.workload(idx, **over)
    check_fwd(gen.generate(cfg), cfg["chunk"])


def test_stiff_impulse_elementwise():
    """Impulse response with d down to 1e-4: elementwise relative error where
    the oracle is >= 1e-30, tiny values elsewhere, no NaN/Inf."""
    cfg = gen.workload(3, H=8, L=4096)
    inp = gen.generate(cfg)
    t = to_device(inp)
    y, hl, ws = pd.pdssm_scan_fwd(t["pi"], t["k"], t["d"], t["b"], t["c"], None, chunk=256)
    y = y.cpu().numpy().astype(np.float64)
    y_ref, _ = oracle.scan_fwd(inp.pi, inp.k, inp.d, inp.b, inp.c, None)
    assert np.isfinite(y).all()
    big = np.abs(y_ref) >= 1e-30
    assert big.sum() > 8
    assert np.max(np.abs(y[big] - y_ref[big]) / np.abs(y_ref[big])) <= 1e-5
    assert np.max(np.abs(y[~big])) <= 1e-30


# ----------------------------------------------------------------------------
# edge cases
# ----------------------------------------------------------------------------
def small(seed, B, H, L, N, K, kind="maps", dtype="f32", per_head=False, h0=True):
    rng = np.random.default_rng(seed)
    nd = H if per_head else 1
    if kind == "maps":
        pi = rng.integers(0, N, size=(nd, K, N))
    elif kind == "perm":
        pi = np.stack([np.stack([rng.permutation(N) for _ in range(K)]) for _ in range(nd)])
    elif kind == "identity":
        pi = np.tile(np.arange(N), (nd, K, 1))
    elif kind == "constant":
        pi = np.stack([np.stack([np.full(N, rng.integers(0, N)) for _ in range(K)])
                       for _ in range(nd)])
    pi = pi.astype(np.int32)
    if not per_head:
        pi = pi[0]
    shape = (B, H, L, N)
    d = rng.uniform(0.5, 1.0, shape).astype(np.float32)
    b = rng.standard_normal(shape).astype(np.float32)
    c = rng.standard_normal(shape).astype(np.float32)
    if dtype == "bf16":
        d, b, c = (gen.round_bf16(x) for x in (d, b, c))
    cfg = dict(dtype=dtype)
    return gen.Inputs(cfg=cfg, pi=pi, d=d, b=b, c=c,
                      k=rng.integers(0, K, size=(B, H, L)).astype(np.int32),
                      h0=rng.standard_normal((B, H, N)).astype(np.float32) if h0 else None,
                      g_y=rng.standard_normal((B, H, L)).astype(np.float32))


@pytest.mark.parametrize("N", [1, 2, 3, 8, 31, 32, 33, 47, 63, 64])
def test_forward_state_sizes(N):
    check_fwd(small(N, 2, 2, 300, N, 5), chunk=37)


@pytest.mark.parametrize("chunk", [1, 2, 7, 16, 17, 100, 999, 1000, 5000])
def test_forward_chunk_sizes(chunk):
    check_fwd(small(chunk, 1, 2, 1000, 24, 6), chunk=chunk)


@pytest.mark.parametrize("kind", ["identity", "constant", "perm"])
@pytest.mark.parametrize("N", [16, 64])
def test_forward_map_kinds(kind, N):
    check_fwd(small(7, 1, 2, 500, N, 3, kind=kind), chunk=64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [32, 64])
def test_permutation_dictionaries_forward_and_adjoint(N, dtype):
    """Every map a permutation: the kernels switch to the permutation step
    (a shuffle for N = 32, one exchange per step for N = 64)."""
    inp = small(40 + N, 2, 2, 700, N, 6, kind="perm", dtype=dtype)
    check_fwd(inp, chunk=96)
    if dtype == "f32":
        check_bwd(inp, chunk=96)


@pytest.mark.parametrize("fan", [7, 8, 9, 20])
@pytest.mark.parametrize("N", [24, 64])
def test_forward_fan_in_around_slot_capacity(fan, N):
    """One target of each map receives exactly `fan` sources; the slot table
    holds up to 8 per target and larger fan-ins take the full scan."""
    inp = small(60 + fan, 1, 2, 300, N, 4)
    rng = np.random.default_rng(fan)
    pi = inp.pi.copy()
    for kk in range(pi.shape[0]):
        row = rng.permutation(N).astype(np.int32)
        row[rng.choice(N, size=fan, replace=False)] = rng.integers(0, N)
        pi[kk] = row
    inp.pi = pi
    check_fwd(inp, chunk=50)
    check_bwd(inp, chunk=50)


def _lane_distance(row, npl):
    """Largest distance in lanes between the first and the last source of one
    target, when the sources, ordered by target, are dealt npl per lane."""
    order = np.argsort(row, kind="stable")
    tg = row[order]
    md, s = 0, 0
    while s < len(tg):
        e = s
        while e + 1 < len(tg) and tg[e + 1] == tg[s]:
            e += 1
        md = max(md, e // npl - s // npl)
        s = e + 1
    return md


def _window_span(row):
    """Largest back-span in lanes of the window table of one N = 64 map
    (None when a fan-in exceeds 8): segments in decreasing fan-in, targets
    ascending within a fan-in, a single-source target moved in front of an
    even-sized segment that would start at an odd entry (at most three
    times), the remaining single-source targets last; two entries per lane."""
    cnt = np.bincount(row, minlength=64)
    if cnt.max() > 8:
        return None
    n1 = int((cnt == 1).sum())
    pos, nins, starts = 0, 0, {}
    for f in range(8, 1, -1):
        tg = [t for t in range(64) if cnt[t] == f]
        if tg and f % 2 == 0 and pos % 2 == 1 and nins < 3 and nins < n1:
            nins += 1
            pos += 1
        for t in tg:
            starts[t] = pos
            pos += f
    span = 0
    for t, s0 in starts.items():
        span = max(span, (s0 + cnt[t] - 1) // 2 - s0 // 2)
    return span


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,fan,levels", [
    (32, 2, 1), (32, 3, 2), (32, 5, 3), (32, 9, 5),
    (64, 3, 0), (64, 5, 0), (64, 6, 0), (64, 7, 2), (64, 9, 3), (64, 17, 5)])
def test_segment_step_shuffle_levels(N, fan, levels, dtype):
    """Maps that are permutations except for one target receiving `fan`
    sources.  The run of that target's sources spans a number of lanes that
    decides how many shuffle levels the segmented sum of the state update
    takes (1, 2, 3 or 5 levels for runs spanning under 2, 4, 8 or 32
    lanes); each case lands in the class named by `levels`.  With N = 64 a
    dictionary whose window tables reach back at most two lanes takes the
    window step instead (levels = 0); fan-ins of 7 and more fall back to the
    segment scan."""
    inp = small(70 + N + fan, 2, 2, 400, N, 5, dtype=dtype)
    rng = np.random.default_rng(N * 100 + fan)
    pi = inp.pi.copy()
    for kk in range(pi.shape[0]):
        row = rng.permutation(N).astype(np.int32)
        sel = rng.choice(N, size=fan, replace=False)
        row[sel] = row[sel[0]]          # that target now has exactly `fan` sources
        pi[kk] = row
    inp.pi = pi
    md = max(_lane_distance(r, N // 32) for r in pi)
    if N == 64:
        spans = [_window_span(r) for r in pi]
        window = all(sp is not None and sp <= 2 for sp in spans)
        assert window == (levels == 0), spans
    if levels:
        assert {1: md < 2, 2: 2 <= md < 4, 3: 4 <= md < 8, 5: md >= 8}[levels], md
    check_fwd(inp, chunk=64)
    check_bwd(inp, chunk=64)


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", ["mixed_fan_in", "no_single_source", "pairs_only",
                                  "fan_in_seven"])
def test_window_step_dictionaries(case, dtype, per_head):
    """N = 64 dictionaries around the window table's limits: maps mixing
    fan-ins 2 to 6 with single-source targets to move in front of
    misaligned even-sized segments, maps with no single-source target at
    all, maps whose targets all have two sources (no segment crosses a
    lane), and maps with one target of fan-in 7 (a back-span of three
    lanes: the segment scan takes over); shared by all heads, or one
    dictionary per head (each warp stages its head's tables)."""
    sizes = {"mixed_fan_in": [6, 5, 4, 4, 3, 2, 2],
             "no_single_source": [6, 5, 5, 4, 4, 3, 3] + [2] * 17,
             "pairs_only": [2] * 32,
             "fan_in_seven": [7, 3, 2]}[case]
    sizes = sizes + [1] * (64 - sum(sizes))
    rng = np.random.default_rng(len(case))
    inp = small(90 + len(case), 2, 2, 333, 64, 6, dtype=dtype, per_head=per_head)
    rows = []
    for _ in range(inp.pi.size // 64):
        targets = rng.permutation(64)[:len(sizes)]
        row = np.concatenate([[t] * f for t, f in zip(targets, sizes)])
        rows.append(row[rng.permutation(64)].astype(np.int32))
    inp.pi = np.stack(rows).reshape(inp.pi.shape)
    spans = [_window_span(r) for r in inp.pi.reshape(-1, 64)]
    assert all(sp is not None and sp <= 2 for sp in spans) == (case != "fan_in_seven"), spans
    check_fwd(inp, chunk=64)
    check_fwd(inp, chunk=128)
    check_bwd(inp, chunk=64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_largest_dictionary_per_head(dtype):
    """The largest sizes the boundary accepts for the scan: N = 64 and
    K = 32 maps per head, a dictionary per head, a ragged last chunk."""
    inp = small(80, 2, 3, 777, 64, 32, dtype=dtype, per_head=True)
    check_fwd(inp, chunk=128)
    check_bwd(inp, chunk=128)


@pytest.mark.parametrize("N", [8, 30, 64])
def test_forward_bf16_aligned_and_unaligned_rows(N):
    check_fwd(small(9, 1, 2, 400, N, 4, dtype="bf16"), chunk=48)


def test_forward_per_head_dictionary_and_K1():
    check_fwd(small(11, 2, 3, 333, 40, 6, per_head=True), chunk=50)
    check_fwd(small(12, 1, 2, 200, 20, 1), chunk=32)


def test_forward_zero_initial_state_and_tiny_lengths():
    check_fwd(small(13, 1, 2, 1, 8, 3, h0=False), chunk=4)
    check_fwd(small(14, 1, 2, 17, 64, 3, h0=False), chunk=4)


def test_forward_empty_sequence():
    inp = small(15, 1, 2, 0, 8, 3)
    t = to_device(inp)
    y, hl, ws = pd.pdssm_scan_fwd(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"], chunk=8)
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert torch.equal(hl, t["h0"])


@pytest.mark.parametrize("single", [False, True])
def test_forward_deterministic(single):
    inp = gen.generate(gen.workload(4, B=1, H=4, L=4096))
    t = to_device(inp)
    fwd = pd.pdssm_scan_fwd_single_pass if single else pd.pdssm_scan_fwd
    y1, h1, _ = fwd(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"], chunk=128)
    y2, h2, _ = fwd(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"], chunk=128)
    assert torch.equal(y1, y2) and torch.equal(h1, h2)


@pytest.mark.parametrize("idx,over,chunk", [(4, dict(B=1, H=4, L=4096), 128),
                                             (1, dict(B=2, H=3, L=1500), 64),
                                             (3, dict(H=4, L=3000), 256)])
def test_backward_deterministic(idx, over, chunk):
    """The adjoint's sums follow fixed trees: two runs give the same bits."""
    inp = gen.generate(gen.workload(idx, **over))
    if inp.k is None:
        inp.k = oracle_k(inp)
    if inp.g_y is None:
        inp.g_y = np.random.default_rng(8).standard_normal(inp.d.shape[:3]).astype(np.float32)
    t = to_device(inp)
    kk = dev(inp.k, torch.int32)
    gy = dev(inp.g_y)
    outs = []
    for _ in range(2):
        y, hl, ws = pd.pdssm_scan_fwd(t["pi"], kk, t["d"], t["b"], t["c"], t["h0"], chunk=chunk,
                                      for_bwd=True)
        g = pd.pdssm_scan_bwd(t["pi"], kk, t["d"], t["b"], t["c"], t["h0"], gy, ws, chunk=chunk)
        outs.append((y, hl) + tuple(g))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


# ----------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------
def check_bwd(inp, chunk, g_hlast=None):
    t = to_device(inp)
    y, hl, ws = pd.pdssm_scan_fwd(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"],
                                  chunk=chunk, for_bwd=True)
    ghl = dev(g_hlast) if g_hlast is not None else None
    g = pd.pdssm_scan_bwd(t["pi"], t["k"], t["d"], t["b"], t["c"], t["h0"], t["g_y"], ws,
                          chunk=chunk, g_hlast=ghl)
    torch.cuda.synchronize()
    assert pd.pdssm_ws_status(ws) == 0
    ref = oracle.scan_bwd(inp.pi, inp.k, inp.d, inp.b, inp.c, inp.h0, inp.g_y, g_hlast)
    tol = tol_for(inp)
    for name, a, r in zip(("g_b", "g_d", "g_c", "g_h0"), g, ref):
        e = floored_relerr(a.cpu().numpy(), r)
        assert e <= tol, f"{name} error {e}"


@pytest.mark.parametrize("N", [1, 5, 32, 33, 64])
def test_backward_state_sizes(N):
    check_bwd(small(20 + N, 1, 2, 300, N, 4), chunk=40)


@pytest.mark.parametrize("chunk", [1, 3, 16, 100, 256])
def test_backward_chunk_sizes(chunk):
    inp = small(30 + chunk, 1, 2, 700, 24, 5)
    rng = np.random.default_rng(chunk)
    check_bwd(inp, chunk, g_hlast=rng.standard_normal((1, 2, 24)).astype(np.float32))


def test_backward_workload_reduced():
    cfg = gen.workload(4, B=1, H=2, L=3000)
    check_bwd(gen.generate(cfg), cfg["chunk"])


def test_backward_bf16_and_maps():
    check_bwd(small(41, 1, 2, 400, 64, 4, dtype="bf16"), chunk=64)
    check_bwd(small(42, 1, 2, 300, 16, 3, kind="constant"), chunk=32)


# ----------------------------------------------------------------------------
# index validation (host-side checks, clamped indices never fault)
# ----------------------------------------------------------------------------
def test_validate_and_clamped_indices_are_reported():
    inp = small(50, 1, 2, 100, 8, 3)
    t = to_device(inp)
    assert pd.pdssm_validate(t["pi"], t["k"], 8) == 0
    bad_k = t["k"].clone()
    bad_k[0, 1, 17] = 3
    assert pd.pdssm_validate(t["pi"], bad_k, 8) == 3
    bad_pi = t["pi"].clone()
    bad_pi[1, 2] = -1
    assert pd.pdssm_validate(bad_pi, t["k"], 8) == 3
    y, hl, ws = pd.pdssm_scan_fwd(t["pi"], bad_k, t["d"], t["b"], t["c"], t["h0"], chunk=16)
    assert pd.pdssm_ws_status(ws) == 3
    assert pd.pdssm_ws_status(ws) == 0
    y, hl, ws = pd.pdssm_scan_fwd(bad_pi, t["k"], t["d"], t["b"], t["c"], t["h0"], chunk=16)
    assert pd.pdssm_ws_status(ws) == 3


@pytest.mark.parametrize("N,kind,H,L,chunk", [
    (64, "maps", 2, 16384, 16),     # 1024 chunks per sequence: clusters of 8 CTAs
    (32, "perm", 4, 8192, 16),      # 512 chunks: clusters of 8
    (24, "maps", 3, 6000, 20),      # 300 chunks: clusters of 4, ragged tail
])
def test_carry_scan_clusters(N, kind, H, L, chunk):
    """Few sequences with many chunks: the carry scans (phase B and bwd B)
    split each sequence over a cluster of CTAs that combine their totals
    through distributed shared memory; the forward, h_last and every
    gradient (g_hlast given, so the adjoint's carry starts non-zero) must
    match the oracle."""
    inp = small(100 + N, 1, H, L, N, 6, kind=kind)
    check_fwd(inp, chunk)
    rng = np.random.default_rng(N)
    check_bwd(inp, chunk, g_hlast=rng.standard_normal((1, H, N)).astype(np.float32))
