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
