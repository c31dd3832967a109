/*
 * Plain CPU oracle for the Flash PD-SSM structured-sparse recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file:
 * only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg load it.
 * It shares no code, header or table with the CUDA library.
 *
 * Everything here is a literal, sequential, fp64 restatement of what the pages
 * fix, written for a reader to check by eye:
 *
 *   Flash PD-SSM (gist.science technical summary, "Methodology" §1, hard
 *   selection): each step scores K dictionary entries with a linear map of
 *   u_t and takes the argmax; the chosen matrix is a one-hot column selector,
 *   so the transition is P_{k_t} diag(d_t) with P[pi(j), j] = 1.
 *
 *     h_t[i] = sum_{j : pi_{k_t}(j) = i} d_t[j] * h_{t-1}[j]  +  b_t[i]
 *     y_t    = sum_i c_t[i] * h_t[i]
 *
 *   The chunk transfer (Methodology §3, phases A-C) is the closed PD form of
 *   the product of a chunk's transitions: a composed index map Pi, the
 *   diagonal product Delta along each column's path, and the chunk's own
 *   state v started from zero.
 *
 *   Exact adjoint (PGF page, "Breaking the Memory Wall", abstract and the
 *   four-stage framework): the reverse recurrence of the same linear system.
 *
 * Conventions (shared by every function):
 *   dims B, H, L, N, K; arrays row-major contiguous.
 *   pi   : int32, entry (h, k, j) at pi[h*pi_hs + k*N + j]   (pi_hs = 0: shared)
 *   k    : int32 [B][H][L]
 *   d,b,c: double [B][H][L][N]
 *   h0   : double [B][H][N] or NULL (NULL means zero)
 *   y    : double [B][H][L];   h_last: double [B][H][N]
 * Indices are assumed valid (the Python wrapper checks them).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX2(a, b, nb) ((a) * (nb) + (b))

/* ---------------------------------------------------------------------------
 * Hard selection.  Logit l_k = sum_d W[h,k,d] * u[b,t,d] evaluated as the fp32
 * chain  acc = 0; for d = 0..D-1: acc = fmaf(W, u, acc)  (single rounding per
 * step, ascending d), then k = the FIRST index of the largest logit (strict >).
 * The pages fix only "linear scores -> argmax"; this fixed fp32 arithmetic is
 * the selection contract both sides implement.
 * u: float [B][L][D] (bf16 inputs arrive already upcast, exactly)
 * W: float [H][K][D]; k_out: int32 [B][H][L]
 * ------------------------------------------------------------------------- */
void oracle_select(int64_t B, int64_t L, int64_t D, int64_t H, int64_t K,
                   const float *u, const float *W, int32_t *k_out)
{
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t t = 0; t < L; ++t) {
            const float *ur = u + (bb * L + t) * D;
            for (int64_t h = 0; h < H; ++h) {
                int32_t best_k = 0;
                float best = 0.0f;
                for (int64_t kk = 0; kk < K; ++kk) {
                    const float *wr = W + (h * K + kk) * D;
                    float acc = 0.0f;
                    for (int64_t q = 0; q < D; ++q)
                        acc = fmaf(wr[q], ur[q], acc);
                    if (kk == 0 || acc > best) {
                        best = acc;
                        best_k = (int32_t)kk;
                    }
                }
                k_out[(bb * H + h) * L + t] = best_k;
            }
        }
}

/* One literal PD step: hn = P_pi diag(dt) h + bt, scatter in ascending source j. */
static void pd_step(int64_t N, const int32_t *pi_k, const double *dt,
                    const double *bt, const double *h, double *hn)
{
    for (int64_t i = 0; i < N; ++i)
        hn[i] = 0.0;
    for (int64_t j = 0; j < N; ++j)
        hn[pi_k[j]] += dt[j] * h[j];
    for (int64_t i = 0; i < N; ++i)
        hn[i] += bt[i];
}

static double dot(int64_t N, const double *a, const double *x)
{
    double s = 0.0;
    for (int64_t i = 0; i < N; ++i)
        s += a[i] * x[i];
    return s;
}

/* ---------------------------------------------------------------------------
 * Forward scan, sequential over t for each (b, h).  y_t reads the state after
 * step t; h_last = h_{L-1} (h_0 when L = 0 is the initial state).
 * ------------------------------------------------------------------------- */
void oracle_scan_fwd(int64_t B, int64_t H, int64_t L, int64_t N, int64_t K,
                     const int32_t *pi, int64_t pi_hs, const int32_t *k,
                     const double *d, const double *b, const double *c,
                     const double *h0, double *y, double *h_last)
{
    (void)K;
    double *h = (double *)malloc(sizeof(double) * (size_t)N);
    double *hn = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t bh = bb * H + hh;
            for (int64_t i = 0; i < N; ++i)
                h[i] = h0 ? h0[bh * N + i] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = (bh * L + t) * N;
                const int32_t *pk = pi + hh * pi_hs + (int64_t)k[bh * L + t] * N;
                pd_step(N, pk, d + row, b + row, h, hn);
                memcpy(h, hn, sizeof(double) * (size_t)N);
                y[bh * L + t] = dot(N, c + row, h);
            }
            if (h_last)
                memcpy(h_last + bh * N, h, sizeof(double) * (size_t)N);
        }
    free(h);
    free(hn);
}

/* ---------------------------------------------------------------------------
 * Chunk transfers in closed PD form.  For the chunk of steps s..e:
 *   h_e = P_Pi diag(Delta) h_{s-1} + v
 * Pi is composed step by step (Pi <- pi_{k_t} o Pi); Delta[j] multiplies, at
 * each step, the d of the coordinate column j currently sits on, before that
 * step's map moves it; v is the chunk's own recurrence started from zero.
 * Outputs per (b, h, chunk): Pi int32, Delta double, v double, each [C][N]
 * with C = ceil(L / chunk); the last chunk may be short.
 * ------------------------------------------------------------------------- */
void oracle_chunk_transfers(int64_t B, int64_t H, int64_t L, int64_t N, int64_t K,
                            const int32_t *pi, int64_t pi_hs, const int32_t *k,
                            const double *d, const double *b, int64_t chunk,
                            int32_t *Pi, double *Delta, double *v)
{
    (void)K;
    const int64_t C = (L + chunk - 1) / chunk;
    double *hn = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t bh = bb * H + hh;
            for (int64_t cc = 0; cc < C; ++cc) {
                int32_t *P = Pi + (bh * C + cc) * N;
                double *Dl = Delta + (bh * C + cc) * N;
                double *vv = v + (bh * C + cc) * N;
                for (int64_t j = 0; j < N; ++j) {
                    P[j] = (int32_t)j;
                    Dl[j] = 1.0;
                    vv[j] = 0.0;
                }
                const int64_t s = cc * chunk;
                const int64_t e = (s + chunk < L) ? s + chunk : L;
                for (int64_t t = s; t < e; ++t) {
                    const int64_t row = (bh * L + t) * N;
                    const int32_t *pk = pi + hh * pi_hs + (int64_t)k[bh * L + t] * N;
                    for (int64_t j = 0; j < N; ++j) {
                        Dl[j] *= d[row + P[j]];
                        P[j] = pk[P[j]];
                    }
                    pd_step(N, pk, d + row, b + row, vv, hn);
                    memcpy(vv, hn, sizeof(double) * (size_t)N);
                }
            }
        }
    free(hn);
}

/* ---------------------------------------------------------------------------
 * Exact adjoint of the forward scan for the loss
 *     l = sum_t g_y[t] * y_t  +  <g_hlast, h_{L-1}>.
 * With M_t = P_{k_t} diag(d_t) and lambda_t = dl/dh_t:
 *     lambda_{L-1} = g_y[L-1] c_{L-1} + g_hlast
 *     lambda_t     = g_y[t] c_t + M_{t+1}^T lambda_{t+1},
 *     (M^T x)[j]   = d[j] * x[pi(j)]
 *     g_b_t = lambda_t,  g_c_t = g_y[t] h_t,
 *     g_d_t[j] = h_{t-1}[j] * lambda_t[pi_{k_t}(j)],
 *     g_h0 = M_0^T lambda_0.
 * The whole state trajectory of one (b, h) is kept (plain, not memory-lean).
 * g_hlast may be NULL (zero).  Outputs: g_b, g_d, g_c [B][H][L][N], g_h0 [B][H][N].
 * ------------------------------------------------------------------------- */
void oracle_scan_bwd(int64_t B, int64_t H, int64_t L, int64_t N, int64_t K,
                     const int32_t *pi, int64_t pi_hs, const int32_t *k,
                     const double *d, const double *b, const double *c,
                     const double *h0, const double *g_y, const double *g_hlast,
                     double *g_b, double *g_d, double *g_c, double *g_h0)
{
    (void)K;
    double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N));
    double *lam = (double *)malloc(sizeof(double) * (size_t)N);
    double *mu = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t bh = bb * H + hh;
            /* hs[t+1] = h_t, hs[0] = h_{-1} = h0 */
            for (int64_t i = 0; i < N; ++i)
                hs[i] = h0 ? h0[bh * N + i] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = (bh * L + t) * N;
                const int32_t *pk = pi + hh * pi_hs + (int64_t)k[bh * L + t] * N;
                pd_step(N, pk, d + row, b + row, hs + t * N, hs + (t + 1) * N);
            }
            /* mu = gradient flowing into h_t from steps after t */
            for (int64_t i = 0; i < N; ++i)
                mu[i] = g_hlast ? g_hlast[bh * N + i] : 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                const int64_t row = (bh * L + t) * N;
                const double gy = g_y[bh * L + t];
                const int32_t *pk = pi + hh * pi_hs + (int64_t)k[bh * L + t] * N;
                for (int64_t i = 0; i < N; ++i) {
                    lam[i] = gy * c[row + i] + mu[i];
                    g_b[row + i] = lam[i];
                    g_c[row + i] = gy * hs[(t + 1) * N + i];
                }
                for (int64_t j = 0; j < N; ++j) {
                    g_d[row + j] = hs[t * N + j] * lam[pk[j]];
                    mu[j] = d[row + j] * lam[pk[j]];
                }
            }
            for (int64_t j = 0; j < N; ++j)
                g_h0[bh * N + j] = (L > 0) ? mu[j] : (g_hlast ? g_hlast[bh * N + j] : 0.0);
        }
    free(hs);
    free(lam);
    free(mu);
}

/* ===========================================================================
 * Dictionary from dense matrices, and the original soft selection.
 *
 * Flash PD-SSM technical summary, Methodology §1: the original PD-SSM forms,
 * at every step, a convex combination of dense dictionary matrices and
 * sparsifies it with a column hardmax (one dense N x N matrix per step);
 * Flash PD-SSM keeps a dictionary of K sparse matrices -- column-hardmax
 * selectors -- and picks one per step by argmax.
 * ========================================================================= */

/* Column hardmax: pi_out[m][j] = first i maximising A[m][i][j] (strict >,
 * ascending i).  A: float [n_mats][N][N]; pi_out: int32 [n_mats][N]. */
void oracle_dict_hardmax(int64_t n_mats, int64_t N, const float *A, int32_t *pi_out)
{
    for (int64_t m = 0; m < n_mats; ++m)
        for (int64_t j = 0; j < N; ++j) {
            const float *Am = A + m * N * N;
            int64_t best_i = 0;
            float best = Am[IDX2(0, j, N)];
            for (int64_t i = 1; i < N; ++i)
                if (Am[IDX2(i, j, N)] > best) {
                    best = Am[IDX2(i, j, N)];
                    best_i = i;
                }
            pi_out[m * N + j] = (int32_t)best_i;
        }
}

/* exp(x) for x <= 0 in fp32, defined step by step so that any IEEE machine
 * with a fused multiply-add computes the same bits: Cody-Waite reduction
 * x = n ln2 + r (ln2 split in two parts), e^r by its Taylor series to degree
 * 7 (Horner, fmaf), times 2^n built from its exponent bits.  Results below
 * 2^-125 are flushed to 0 (x < -86).  Relative error below 2e-7 (Taylor
 * remainder (ln2/2)^8 / 8! < 1.5e-9 plus the roundings). */
float oracle_soft_exp(float x)
{
    if (x < -86.0f)
        return 0.0f;
    const float n = rintf(x * 1.44269504f);
    float r = fmaf(-n, 0.693145751953125f, x);
    r = fmaf(-n, 1.42860677e-06f, r);
    float p = 1.0f / 5040.0f;
    p = fmaf(p, r, 1.0f / 720.0f);
    p = fmaf(p, r, 1.0f / 120.0f);
    p = fmaf(p, r, 1.0f / 24.0f);
    p = fmaf(p, r, 1.0f / 6.0f);
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    const int32_t e = (int32_t)n + 127;
    float two_n;
    const uint32_t bits = (uint32_t)e << 23;
    memcpy(&two_n, &bits, 4);
    return p * two_n;
}

/* Soft-selection weights of one step, in fp32: m = max_k l_k, e_k =
 * oracle_soft_exp((l_k - m) * inv_tau), Z = sum_k e_k (ascending k),
 * s_k = e_k / Z.  A convex combination (the s_k are >= 0, sum ~ 1). */
static void soft_weights(int64_t K, const float *l, float inv_tau, float *s)
{
    float m = l[0];
    for (int64_t k = 1; k < K; ++k)
        if (l[k] > m)
            m = l[k];
    float Z = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        s[k] = oracle_soft_exp((l[k] - m) * inv_tau);
        Z += s[k];
    }
    for (int64_t k = 0; k < K; ++k)
        s[k] = s[k] / Z;
}

/* The original PD-SSM transition of every step: logits l_k = the fp32 fmaf
 * chain of W[h][k] . u[b][t] (as in oracle_select), weights s = the soft
 * weights above, the dense combination M[i][j] = sum_k s_k A_k[i][j]
 * (fp32, acc = fmaf(s_k, A_k[i][j], acc) over ascending k from 0), and its
 * column hardmax maps_out[b][h][t][j] = first i maximising M[i][j].
 * u: float [B][L][D]; W: float [H][K][D]; A: float, matrix (h, k) at
 * A + h*a_hs + k*N*N (a_hs = 0: shared by the heads). */
void oracle_soft_maps(int64_t B, int64_t L, int64_t D, int64_t H, int64_t K, int64_t N,
                      const float *u, const float *W, const float *A, int64_t a_hs,
                      float inv_tau, int32_t *maps_out)
{
    float *l = (float *)malloc(sizeof(float) * (size_t)K);
    float *s = (float *)malloc(sizeof(float) * (size_t)K);
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t t = 0; t < L; ++t) {
                const float *ur = u + (bb * L + t) * D;
                for (int64_t kk = 0; kk < K; ++kk) {
                    const float *wr = W + (h * K + kk) * D;
                    float acc = 0.0f;
                    for (int64_t q = 0; q < D; ++q)
                        acc = fmaf(wr[q], ur[q], acc);
                    l[kk] = acc;
                }
                soft_weights(K, l, inv_tau, s);
                int32_t *out = maps_out + ((bb * H + h) * L + t) * N;
                for (int64_t j = 0; j < N; ++j) {
                    int64_t best_i = 0;
                    float best = 0.0f;
                    for (int64_t i = 0; i < N; ++i) {
                        float acc = 0.0f;
                        for (int64_t kk = 0; kk < K; ++kk)
                            acc = fmaf(s[kk], A[h * a_hs + kk * N * N + IDX2(i, j, N)], acc);
                        if (i == 0 || acc > best) {
                            best = acc;
                            best_i = i;
                        }
                    }
                    out[j] = (int32_t)best_i;
                }
            }
    free(l);
    free(s);
}

/* Forward scan with one map per step (the original PD-SSM's input-dependent
 * selectors): as oracle_scan_fwd with pi_{k_t} replaced by maps[b][h][t]. */
void oracle_scan_fwd_maps(int64_t B, int64_t H, int64_t L, int64_t N, const int32_t *maps,
                          const double *d, const double *b, const double *c,
                          const double *h0, double *y, double *h_last)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)N);
    double *hn = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t bh = bb * H + hh;
            for (int64_t i = 0; i < N; ++i)
                h[i] = h0 ? h0[bh * N + i] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = (bh * L + t) * N;
                pd_step(N, maps + row, d + row, b + row, h, hn);
                memcpy(h, hn, sizeof(double) * (size_t)N);
                y[bh * L + t] = dot(N, c + row, h);
            }
            if (h_last)
                memcpy(h_last + bh * N, h, sizeof(double) * (size_t)N);
        }
    free(h);
    free(hn);
}

/* ===========================================================================
 * Straight-through surrogate gradients of the selection and the dictionary.
 *
 * Flash PD-SSM technical summary, Methodology §2: the forward uses the hard
 * selection (argmax) and the hard dictionary (column hardmax); the backward
 * replaces the discrete choices by tempered softmaxes so that gradients reach
 * the selection weights and the dense dictionary matrices (Proposition 2's
 * surrogate gradients, exact as tau -> 0; its expressions are not on the
 * pages).  Reading taken here: each discrete choice is relaxed on its own,
 * the other one held at its hard value, around the hard trajectory
 * (lambda_t = dl/dh_t of the hard model, oracle_scan_bwd's g_b, and
 * z_t = d_t (.) h_{t-1}):
 *   selection:  T_t = sum_k s_{t,k} P_k,  s_t = softmax(l_t * inv_tau_s),
 *               P_k the hard dictionary (column hardmax of A_k):
 *     g_s[t,k] = lambda_t^T P_k z_t = sum_j lambda_t[pi_k(j)] z_t[j]
 *     g_l[t,k] = inv_tau_s s_{t,k} (g_s[t,k] - sum_k' s_{t,k'} g_s[t,k'])
 *     g_W[h,k,:] = sum_{b,t} g_l[b,h,t,k] u[b,t,:]
 *   dictionary: T_t = Q_{k_t},  Q_k[:, j] = softmax(A_k[:, j] * inv_tau_a)
 *               (column softmax), k_t the hard selection:
 *     G_k = sum_{b,h,t : k_t = k} lambda_t z_t^T        (per head if a_hs != 0)
 *     g_A[k][:,j] = inv_tau_a Q_k[:,j] (.) (G_k[:,j] - <Q_k[:,j], G_k[:,j]>).
 * These are exactly the gradients, at fixed lambda and z, of the linearised
 * losses G_sel(W) = sum_t lambda_t^T (sum_k s_{t,k} P_k) z_t and
 * G_dict(A) = sum_t lambda_t^T Q_{k_t} z_t.  Both keep the backward sparse:
 * O(N K) per step for the selection, one O(N^2) outer product per step for
 * the dictionary.  fp64 throughout except the logits (the fp32 fmaf chain of
 * oracle_select, which also gives k_t) and the hard dictionary
 * (oracle_dict_hardmax of A).
 * Loss: sum_t g_y[t] y_t + <g_hlast, h_{L-1}> (g_hlast may be NULL).
 * Outputs: g_l double [B][H][L][K], g_W double [H][K][D],
 * g_A double [Hd][K][N][N] with Hd = H if a_hs else 1.
 * ========================================================================= */
void oracle_surrogate_grad(int64_t B, int64_t H, int64_t L, int64_t N, int64_t K, int64_t D,
                           const float *u, const float *W, const float *A, int64_t a_hs,
                           double inv_tau_s, double inv_tau_a, const double *d,
                           const double *b, const double *c, const double *h0,
                           const double *g_y, const double *g_hlast, double *g_l,
                           double *g_W, double *g_A)
{
    const int64_t Hd = a_hs ? H : 1;
    const int64_t NN = N * N;
    /* hard dictionary, and the column softmaxes of the dictionary matrices */
    int32_t *pi = (int32_t *)malloc(sizeof(int32_t) * (size_t)(Hd * K * N));
    oracle_dict_hardmax(Hd * K, N, A, pi);
    double *Q = (double *)malloc(sizeof(double) * (size_t)(Hd * K * NN));
    for (int64_t m = 0; m < Hd * K; ++m)
        for (int64_t j = 0; j < N; ++j) {
            const float *Am = A + (m / K) * a_hs + (m % K) * NN;
            double mx = (double)Am[IDX2(0, j, N)];
            for (int64_t i = 1; i < N; ++i)
                if ((double)Am[IDX2(i, j, N)] > mx)
                    mx = (double)Am[IDX2(i, j, N)];
            double Z = 0.0;
            for (int64_t i = 0; i < N; ++i) {
                Q[m * NN + IDX2(i, j, N)] = exp(((double)Am[IDX2(i, j, N)] - mx) * inv_tau_a);
                Z += Q[m * NN + IDX2(i, j, N)];
            }
            for (int64_t i = 0; i < N; ++i)
                Q[m * NN + IDX2(i, j, N)] /= Z;
        }
    /* hard selection, the hard trajectory and its adjoint */
    int32_t *k = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B * H * L));
    oracle_select(B, L, D, H, K, u, W, k);
    double *g_b = (double *)malloc(sizeof(double) * (size_t)(B * H * L * N));
    double *g_d = (double *)malloc(sizeof(double) * (size_t)(B * H * L * N));
    double *g_c = (double *)malloc(sizeof(double) * (size_t)(B * H * L * N));
    double *g_h0 = (double *)malloc(sizeof(double) * (size_t)(B * H * N));
    oracle_scan_bwd(B, H, L, N, K, pi, a_hs ? K * N : 0, k, d, b, c, h0, g_y, g_hlast, g_b,
                    g_d, g_c, g_h0);
    double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N));
    double *lv = (double *)malloc(sizeof(double) * (size_t)K);
    double *s = (double *)malloc(sizeof(double) * (size_t)K);
    double *gs = (double *)malloc(sizeof(double) * (size_t)K);
    double *z = (double *)malloc(sizeof(double) * (size_t)N);
    double *G = (double *)calloc((size_t)(Hd * K * NN), sizeof(double));
    for (int64_t i = 0; i < H * K * D; ++i)
        g_W[i] = 0.0;
    for (int64_t bb = 0; bb < B; ++bb)
        for (int64_t hh = 0; hh < H; ++hh) {
            const int64_t bh = bb * H + hh;
            const int64_t hd = a_hs ? hh : 0;
            for (int64_t i = 0; i < N; ++i)
                hs[i] = h0 ? h0[bh * N + i] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = (bh * L + t) * N;
                const int32_t *pk = pi + hd * K * N + (int64_t)k[bh * L + t] * N;
                pd_step(N, pk, d + row, b + row, hs + t * N, hs + (t + 1) * N);
            }
            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = (bh * L + t) * N;
                const double *lam = g_b + row;
                const float *ur = u + (bb * L + t) * D;
                for (int64_t j = 0; j < N; ++j)
                    z[j] = d[row + j] * hs[t * N + j];
                /* selection: logits in the fp32 contract, softmax in fp64 */
                double mx = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) {
                    const float *wr = W + (hh * K + kk) * D;
                    float acc = 0.0f;
                    for (int64_t q = 0; q < D; ++q)
                        acc = fmaf(wr[q], ur[q], acc);
                    lv[kk] = (double)acc;
                    if (kk == 0 || lv[kk] > mx)
                        mx = lv[kk];
                }
                double Z = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) {
                    s[kk] = exp((lv[kk] - mx) * inv_tau_s);
                    Z += s[kk];
                }
                for (int64_t kk = 0; kk < K; ++kk)
                    s[kk] /= Z;
                double sg = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) {
                    const int32_t *pq = pi + hd * K * N + kk * N;
                    double acc = 0.0;
                    for (int64_t j = 0; j < N; ++j)
                        acc += lam[pq[j]] * z[j];
                    gs[kk] = acc;
                    sg += s[kk] * acc;
                }
                for (int64_t kk = 0; kk < K; ++kk) {
                    const double gl = inv_tau_s * s[kk] * (gs[kk] - sg);
                    g_l[(bh * L + t) * K + kk] = gl;
                    for (int64_t q = 0; q < D; ++q)
                        g_W[(hh * K + kk) * D + q] += gl * (double)ur[q];
                }
                /* dictionary: the outer product joins the selected matrix's sum */
                double *Gk = G + (hd * K + k[bh * L + t]) * NN;
                for (int64_t i = 0; i < N; ++i)
                    for (int64_t j = 0; j < N; ++j)
                        Gk[IDX2(i, j, N)] += lam[i] * z[j];
            }
        }
    for (int64_t m = 0; m < Hd * K; ++m)
        for (int64_t j = 0; j < N; ++j) {
            double dotq = 0.0;
            for (int64_t i = 0; i < N; ++i)
                dotq += Q[m * NN + IDX2(i, j, N)] * G[m * NN + IDX2(i, j, N)];
            for (int64_t i = 0; i < N; ++i)
                g_A[m * NN + IDX2(i, j, N)] =
                    inv_tau_a * Q[m * NN + IDX2(i, j, N)] * (G[m * NN + IDX2(i, j, N)] - dotq);
        }
    free(pi);
    free(Q);
    free(k);
    free(g_b);
    free(g_d);
    free(g_c);
    free(g_h0);
    free(hs);
    free(lv);
    free(s);
    free(gs);
    free(z);
    free(G);
}

/* oracle_soft_exp over an array (for the tests). */
void oracle_soft_exp_array(int64_t n, const float *x, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_soft_exp(x[i]);
}
