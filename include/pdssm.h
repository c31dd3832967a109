/*
 * pdssm.h -- C ABI of the B200 (sm_100a) Flash PD-SSM scan library.
 *
 * The recurrence (Flash PD-SSM technical summary, Methodology §1 "hard
 * selection", one-hot column selector):
 *
 *     k_t    = argmax_k (W_sel u_t)_k
 *     h_t    = P_{k_t} diag(d_t) h_{t-1} + b_t,   P_k[pi_k(j), j] = 1
 *     y_t    = <c_t, h_t>
 *
 * per (batch b, head h), evaluated as a chunked scan in three phases
 * (Methodology §3: A chunk-local recurrence, B carry prefix scan, C carry
 * correction), with its exact adjoint (Breaking the Memory Wall / PGF,
 * abstract: exact analytical derivatives by chunked evolution, memory
 * independent of L apart from per-chunk carries).
 *
 * Conventions for every call
 * --------------------------
 *  * All tensor pointers are DEVICE pointers to caller-owned, row-major,
 *    contiguous memory.  The library allocates nothing and keeps no state
 *    between calls; scratch lives in the caller's workspace `ws` (the one
 *    exception, pdssm_scan_fwd_noalloc, uses a fixed array inside the
 *    library instead, described there).
 *  * Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  A returned PDSSM_OK means the kernels were launched;
 *    device-side problems are recorded in the workspace status word and read
 *    back with pdssm_ws_status().  pdssm_validate() and pdssm_ws_status()
 *    synchronise the stream.
 *  * Consecutive kernels may overlap (programmatic dependent launch): a
 *    kernel of this library can start while the previous kernel on the
 *    stream, when that is one of this library's, is finishing.  Before it
 *    waits for that kernel it reads only the inputs u, W_sel, d, b, c of its
 *    own call, so these must not be outputs of the immediately preceding
 *    call; inputs written by the caller's own kernels or copies are safe
 *    (those complete first).
 *  * Shapes:   u [B][L][D_in]        W_sel [H][K][D_in] (fp32)
 *              pi_dict: entry (h,k,j) at pi_dict[h*pi_head_stride + k*N + j]
 *                       (pi_head_stride = 0: one [K][N] dictionary for all heads,
 *                        = K*N: one per head)
 *              k [B][H][L] int32      d, b, c [B][H][L][N] (fp32 or bf16)
 *              h0, h_last [B][H][N] fp32     y [B][H][L] fp32
 *              g_y [B][H][L] fp32     g_b, g_d, g_c [B][H][L][N] fp32
 *              g_hlast, g_h0 [B][H][N] fp32
 *  * Limits: 1 <= N <= 64, 1 <= K <= 32, 1 <= D_in <= 256, chunk >= 1,
 *    B, H >= 1, L >= 0.  L need not be a multiple of chunk.
 *  * Errors: NULL required pointers, bad sizes or a too-small workspace give
 *    PDSSM_ERR_INVALID_ARG / PDSSM_ERR_WORKSPACE before anything is launched;
 *    sizes beyond the limits give PDSSM_ERR_UNSUPPORTED; a failed launch
 *    gives PDSSM_ERR_CUDA.  Out-of-range k or pi values are clamped by the
 *    kernels (memory-safe) and flagged PDSSM_ERR_BAD_INDEX in the status word;
 *    pdssm_validate() checks them up front.
 */
#ifndef PDSSM_H
#define PDSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pdssm_dims {
    int64_t B, H, L, N, K, D_in;   /* D_in is used by pdssm_select only */
} pdssm_dims;

typedef enum pdssm_dtype { PDSSM_F32 = 0, PDSSM_BF16 = 1 } pdssm_dtype;

typedef enum pdssm_status {
    PDSSM_OK = 0,
    PDSSM_ERR_INVALID_ARG = 1,
    PDSSM_ERR_UNSUPPORTED = 2,
    PDSSM_ERR_BAD_INDEX = 3,
    PDSSM_ERR_CUDA = 4,
    PDSSM_ERR_TIMEOUT = 5,
    PDSSM_ERR_WORKSPACE = 6
} pdssm_status;

/* Human-readable name of a status code.  Never NULL. */
const char *pdssm_status_str(int status);

/* Text of the last error seen by a call on this host thread ("" if none).
 * Owned by the library; valid until the next call on the same thread. */
const char *pdssm_last_error(void);

/* Library ABI version (major * 100 + minor). */
int pdssm_version(void);

/*
 * Workspace bytes needed by pdssm_scan_fwd (for_bwd = 0) or by the pair
 * pdssm_scan_fwd + pdssm_scan_bwd (for_bwd = 1) at these sizes.  The
 * workspace holds a sanitised copy of the dictionary (phase A0), the chunk
 * transfers (Pi_c, Delta_c, v_c), the carries H_c and a status word:
 * O(B*H*ceil(L/chunk)*N), i.e. 1/chunk of the size of d.  Returns 0 when the
 * arguments are invalid.  Pure host function.
 */
size_t pdssm_workspace_bytes(const pdssm_dims *dims, int64_t pi_head_stride,
                             int64_t chunk, int for_bwd);

/*
 * Hard selection (Flash PD-SSM technical summary, Methodology §1): for every
 * (b, h, t),  k_out[b][h][t] = first index of the largest logit
 *     l_k = sum_{q < D_in} W_sel[h][k][q] * u[b][t][q],
 * each logit evaluated as the fp32 chain acc = fmaf(W, u, acc) in ascending q
 * from acc = 0 (bf16 u is upcast exactly).  This fixed arithmetic makes k
 * reproducible bit for bit on any IEEE machine.
 * u: device [B][L][D_in] of u_dtype; W_sel: device fp32 [H][K][D_in];
 * k_out: device int32 [B][H][L].  Needs no workspace.
 */
pdssm_status pdssm_select(const pdssm_dims *dims, const void *u,
                          pdssm_dtype u_dtype, const float *W_sel,
                          int32_t *k_out, void *stream);

/* Arithmetic route of the hard selection (pdssm_select_with). */
typedef enum pdssm_select_method {
    PDSSM_SELECT_AUTO = 0,         /* tensor cores where they apply, else the fma chain */
    PDSSM_SELECT_FMA_CHAIN = 1,    /* the fp32 fma chain on the CUDA cores, any shape */
    PDSSM_SELECT_TENSOR_CORE = 2   /* tcgen05 logits + certified argmax; bf16 u, D_in a
                                      multiple of 16, K a power of two, H*K <= 256,
                                      else PDSSM_ERR_UNSUPPORTED */
} pdssm_select_method;

/*
 * pdssm_select with an explicit arithmetic route.  Every route returns the
 * same k, bit for bit: the tensor-core route bounds the error of its logits
 * (see pdssm_select_tc_logits), keeps every index within twice that bound of
 * the top logit as a candidate, and decides several candidates with the
 * contract's fma chains.  `method` is a pdssm_select_method.
 */
pdssm_status pdssm_select_with(const pdssm_dims *dims, const void *u,
                               pdssm_dtype u_dtype, const float *W_sel,
                               int32_t *k_out, int method, void *stream);

/*
 * Test hook of the tensor-core selection: runs pdssm_select_with(...,
 * PDSSM_SELECT_TENSOR_CORE) on bf16 u and also writes, per row r = b*L + t,
 *     logits_out[r][h*K + k] = the tensor-core logit (bf16 u times the
 *                              bf16 hi and lo parts of W_sel, fp32 sums),
 *     scale_out[r][h]        = ||u_r||_2 * max_k ||W_sel[h][k]||_2, rounded up.
 * The selection treats |logit - exact sum| <= (D_in 2^-21 + 2^-16) scale as
 * the tensor cores' error bound; this hook lets a test check that bound
 * against exact sums.  logits_out: device fp32 [B*L][H*K]; scale_out: device
 * fp32 [B*L][H].
 */
pdssm_status pdssm_select_tc_logits(const pdssm_dims *dims, const void *u,
                                    const float *W_sel, int32_t *k_out,
                                    float *logits_out, float *scale_out,
                                    void *stream);

/*
 * Chunked forward scan (Methodology §3).  Runs phase A0 (sanitised copy of
 * the dictionary), A (per chunk: local readout of the state started from zero,
 * closed PD transfer Pi_c, Delta_c, v_c), B (carry prefix scan H_c, h_last)
 * and C (carry correction of the readout y), as three kernels.  Writes y [B][H][L] and, when
 * non-NULL, h_last [B][H][N] = h_{L-1} (h0 when L = 0).  h0 may be NULL
 * (zero initial state).  ws must hold pdssm_workspace_bytes(dims,
 * pi_head_stride, chunk, 0) bytes, 256-byte aligned; its contents are
 * overwritten.  d, b, c share in_dtype.
 */
pdssm_status pdssm_scan_fwd(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k,
                            const void *d, const void *b, const void *c,
                            pdssm_dtype in_dtype, const float *h0, float *y,
                            float *h_last, int64_t chunk, void *ws,
                            size_t ws_bytes, void *stream);

/*
 * Exact adjoint of pdssm_scan_fwd (PGF: reverse evolution, per-chunk
 * recompute) for the loss  sum_t g_y[t] y_t + <g_hlast, h_last>:
 *     lambda_t = g_y[t] c_t + M_{t+1}^T lambda_{t+1},  (M^T x)[j] = d[j] x[pi(j)]
 *     g_b_t = lambda_t,  g_c_t = g_y[t] h_t,
 *     g_d_t[j] = h_{t-1}[j] lambda_t[pi_{k_t}(j)],  g_h0 = M_0^T lambda_0.
 * Must follow pdssm_scan_fwd on the same stream with identical arguments and
 * the SAME workspace, untouched in between, sized with for_bwd = 1: the
 * forward's chunk transfers and carries are the backward's checkpoints; h is
 * recomputed inside each chunk.  g_hlast may be NULL (zero).  g_h0 may be
 * NULL (not written).  Writes g_b, g_d, g_c and g_h0 (fp32).
 */
pdssm_status pdssm_scan_bwd(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k,
                            const void *d, const void *b, const void *c,
                            pdssm_dtype in_dtype, const float *h0,
                            const float *g_y, const float *g_hlast,
                            float *g_b, float *g_d, float *g_c, float *g_h0,
                            int64_t chunk, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * Kernel-level timing of one call (a measurement aid, not part of the
 * method).  The caller supplies created cudaEvent_t handles; the traced
 * calls record events[i] on the stream just before the i-th kernel they
 * launch and events[n_kernels] after the last, and name each kernel in
 * names[i] (static strings).  Events recorded between the kernels keep them
 * from overlapping (no programmatic dependent launch across an event), so
 * traced calls run slightly slower than untraced ones.
 */
#define PDSSM_TRACE_MAX_KERNELS 8
typedef struct pdssm_trace {
    void *const *events;   /* in: max_events cudaEvent_t handles */
    int max_events;        /* in: >= 2 */
    int n_kernels;         /* out */
    const char *names[PDSSM_TRACE_MAX_KERNELS];   /* out */
} pdssm_trace;

/* pdssm_scan_fwd, recording `trace` (see above).  Same results. */
pdssm_status pdssm_scan_fwd_traced(const pdssm_dims *dims,
                                   const int32_t *pi_dict,
                                   int64_t pi_head_stride, const int32_t *k,
                                   const void *d, const void *b,
                                   const void *c, pdssm_dtype in_dtype,
                                   const float *h0, float *y, float *h_last,
                                   int64_t chunk, void *ws, size_t ws_bytes,
                                   void *stream, pdssm_trace *trace);

/*
 * Hard selection inside the forward scan (Flash PD-SSM technical summary,
 * Methodology §1 and §4: the selection of step t is the argmax of K linear
 * scores of u_t): the results of pdssm_select followed by pdssm_scan_fwd,
 * in one single-pass kernel whose CTAs select their own chunk's steps, so
 * the indices never travel through device memory (k_out, when not NULL,
 * receives a copy for a later backward).  The selection follows the
 * contract of pdssm_select bit for bit: logits of a warp-level bf16 tensor-
 * core product against W_sel's hi / lo bf16 parts, a certified argmax, and
 * the exact fp32 fma chains for near ties.  Needs bf16 u, D_in a multiple of
 * 16 (<= 256), K <= 16, N = 32 or 64 with 16-byte aligned rows, chunk <=
 * 1024 and L >= 1; otherwise PDSSM_ERR_UNSUPPORTED (use the two calls).
 * Other arguments as pdssm_scan_fwd (dims->D_in is u's width).
 */
pdssm_status pdssm_select_scan_fwd(const pdssm_dims *dims, const void *u,
                                   pdssm_dtype u_dtype, const float *W_sel,
                                   const int32_t *pi_dict,
                                   int64_t pi_head_stride, const void *d,
                                   const void *b, const void *c,
                                   pdssm_dtype in_dtype, const float *h0,
                                   float *y, float *h_last, int32_t *k_out,
                                   int64_t chunk, void *ws, size_t ws_bytes,
                                   void *stream);

/*
 * The forward scan as ONE kernel (Methodology §3 with the three phases
 * fused): persistent CTAs take chunks in chunk order; a team of warps runs
 * phase A on the chunk's sub-chunks, composes their transfers, publishes
 * the chunk's transfer, takes its carry from the predecessors' published
 * transfers and carries (decoupled look-back, every wait bounded), publishes
 * its own carry, and runs phase C on data phase A read shortly before.
 * Same arguments, results and workspace contents as pdssm_scan_fwd (so
 * pdssm_scan_bwd may follow it); needs N = 32 or 64 with 16-byte aligned
 * rows, else PDSSM_ERR_UNSUPPORTED.  It moves close to the algorithmic bytes
 * (no phase C re-read from DRAM for most chunks) but, with thousands of
 * chunks in flight over few sequences, spends more time on the look-back
 * chain than the carry scan of the three-kernel form, which stays the
 * default.
 */
pdssm_status pdssm_scan_fwd_single_pass(const pdssm_dims *dims,
                                        const int32_t *pi_dict,
                                        int64_t pi_head_stride,
                                        const int32_t *k, const void *d,
                                        const void *b, const void *c,
                                        pdssm_dtype in_dtype, const float *h0,
                                        float *y, float *h_last, int64_t chunk,
                                        void *ws, size_t ws_bytes, void *stream);

/* pdssm_scan_bwd, recording `trace` (see above).  Same results. */
pdssm_status pdssm_scan_bwd_traced(const pdssm_dims *dims,
                                   const int32_t *pi_dict,
                                   int64_t pi_head_stride, const int32_t *k,
                                   const void *d, const void *b,
                                   const void *c, pdssm_dtype in_dtype,
                                   const float *h0, const float *g_y,
                                   const float *g_hlast, float *g_b,
                                   float *g_d, float *g_c, float *g_h0,
                                   int64_t chunk, void *ws, size_t ws_bytes,
                                   void *stream, pdssm_trace *trace);

/*
 * Dictionary from dense matrices (Flash PD-SSM technical summary,
 * Methodology §1: the dictionary holds column one-hot selectors, the column
 * hardmax of dense matrices):
 *     pi_out[m][j] = first i maximising A[m][i][j]   (strict >, ascending i)
 * for the n_mats matrices A [n_mats][N][N] (fp32, device); pi_out int32
 * [n_mats][N] (device) is then a dictionary for pdssm_scan_fwd (n_mats = K,
 * or H*K with pi_head_stride = K*N).  1 <= N <= 64.
 */
pdssm_status pdssm_dict_hardmax(int64_t n_mats, int64_t N, const float *A,
                                int32_t *pi_out, void *stream);

/*
 * The original PD-SSM's input-dependent transitions (Methodology §1: a
 * convex combination of dense dictionary matrices, sparsified by a column
 * hardmax), as a dense comparison path for the hard selection.  For every
 * (b, h, t), in this fixed fp32 arithmetic:
 *   l_k  = the fma chain of pdssm_select (W_sel[h][k] . u[b][t], ascending q),
 *   m    = max_k l_k,  e_k = exp_soft((l_k - m) * inv_tau),  Z = sum_k e_k
 *          (ascending k),  s_k = e_k / Z,
 *   M[i][j] = fmaf chain over ascending k of s_k * A_k[i][j] (from 0),
 *   maps_out[b][h][t][j] = first i maximising M[i][j],
 * where exp_soft(x) (x <= 0) is Cody-Waite reduction x = n ln2 + r (ln2 as
 * 0.693145751953125 + 1.42860677e-06), the degree-7 Taylor polynomial of e^r
 * in Horner form with fmaf, times 2^n; 0 for x < -86.  Dictionary matrix
 * (h, k) at A + h*a_head_stride + k*N*N (a_head_stride = 0: shared by the
 * heads).  u [B][L][D_in] (fp32 or bf16), W_sel [H][K][D_in] fp32, A fp32,
 * maps_out int32 [B][H][L][N], all device.  Costs O(N^2 K) per step.
 */
pdssm_status pdssm_soft_maps(const pdssm_dims *dims, const void *u,
                             pdssm_dtype u_dtype, const float *W_sel,
                             const float *A, int64_t a_head_stride,
                             float inv_tau, int32_t *maps_out, void *stream);

/*
 * Forward scan with one column-selector map per step (the transitions of
 * pdssm_soft_maps): as pdssm_scan_fwd with pi_{k_t} replaced by
 * maps[b][h][t] (int32 [B][H][L][N], entries in [0, N)).  Sequential in t,
 * one warp per (b, h); needs no workspace.  y [B][H][L] and h_last [B][H][N]
 * (may be NULL) fp32; h0 may be NULL.
 */
pdssm_status pdssm_scan_fwd_maps(const pdssm_dims *dims, const int32_t *maps,
                                 const void *d, const void *b, const void *c,
                                 pdssm_dtype in_dtype, const float *h0,
                                 float *y, float *h_last, void *stream);

/*
 * Straight-through surrogate gradients of the hard selection and of the
 * column-hardmax dictionary (Flash PD-SSM technical summary, Methodology
 * §2: hard forward; in the backward the discrete choices are replaced by
 * tempered softmaxes so that gradients reach the selection weights W_sel
 * and the dense dictionary matrices A; the pages do not print Proposition
 * 2's expressions).  Reading: each choice is relaxed on its own around the
 * hard trajectory, with lambda_t = dl/dh_t (pdssm_scan_bwd's g_b) and
 * z_t = d_t (.) h_{t-1}:
 *   selection  (softmax over the hard selectors P_k, weights
 *               s_t = softmax(l_t * inv_tau_s), l_t the logits of pdssm_select):
 *     g_s[t,k]    = sum_j lambda_t[pi_k(j)] z_t[j]
 *     g_logits[b][h][t][k] = inv_tau_s s_k (g_s[t,k] - sum_k' s_k' g_s[t,k'])
 *     g_W[h][k][:] = sum_{b,t} g_logits[b][h][t][k] u[b][t][:]
 *   dictionary (column softmax Q_k of A_k * inv_tau_a for the selected k_t):
 *     G_k = sum_{b,h,t : k_t = k} lambda_t z_t^T
 *     g_A[k][:,j] = inv_tau_a Q_k[:,j] (.) (G_k[:,j] - <Q_k[:,j], G_k[:,j]>)
 * The costs stay those of the hard model: O(N K) per step for the selection,
 * one N x N outer product per step for the dictionary.
 * Preconditions (same dims, chunk, dictionary): pi_dict = pdssm_dict_hardmax
 * of A ([Hd][K][N], Hd = H when a_head_stride = K*N*N, else 1); k = the hard
 * selection; pdssm_scan_fwd ran with workspace `ws` (its carries are read)
 * and pi_head_stride = K*N when A is per head; lambda = g_b of
 * pdssm_scan_bwd.  u [B][L][D_in] (fp32 / bf16), W_sel [H][K][D_in] fp32,
 * A fp32 (matrix (h, k) at A + h*a_head_stride + k*N*N), d, b of in_dtype,
 * h0 fp32 or NULL.  Outputs fp32: g_logits [B][H][L][K], g_W [H][K][D_in],
 * g_A like A.  scratch: pdssm_surrogate_scratch_bytes(dims, a_head_stride)
 * bytes, 256-byte aligned.  Deterministic (every sum in a fixed order).
 */
size_t pdssm_surrogate_scratch_bytes(const pdssm_dims *dims,
                                     int64_t a_head_stride);
pdssm_status pdssm_surrogate_bwd(const pdssm_dims *dims, const void *u,
                                 pdssm_dtype u_dtype, const float *W_sel,
                                 const float *A, int64_t a_head_stride,
                                 const int32_t *pi_dict, const int32_t *k,
                                 const void *d, const void *b,
                                 pdssm_dtype in_dtype, const float *h0,
                                 const float *lambda, int64_t chunk,
                                 const void *ws, size_t ws_bytes,
                                 float inv_tau_s, float inv_tau_a,
                                 void *scratch, size_t scratch_bytes,
                                 float *g_logits, float *g_W, float *g_A,
                                 void *stream);

/*
 * pdssm_scan_fwd for callers that cannot allocate device memory.  The pages
 * have no counterpart of this call: it exists for host code that owns no
 * allocator (device memory held by another framework's pool), must not call
 * cudaMalloc in its loop (the call can synchronise the device), or runs
 * where allocation after start-up is forbidden.  Same arguments and results
 * as pdssm_scan_fwd without `ws`: the workspace is a file-scope device array
 * of pdssm_noalloc_scratch_bytes() bytes (4 MiB) that every GPU loading the
 * library holds until the process exits; nothing is allocated.
 *  * Sizes whose workspace (pdssm_workspace_bytes(..., 0)) exceeds that
 *    maximum return PDSSM_ERR_UNSUPPORTED before anything is launched.
 *  * The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture.
 *  * Every call on a device shares the one array and it keeps the last
 *    call's contents (each call resets what must start at zero).  Calls whose
 *    work overlaps on the GPU (different streams, no ordering) race on it.
 *  * The device status word of these calls lives in the shared array; read
 *    it with pdssm_noalloc_status.
 *  * The array's address is remembered per device for the life of the
 *    process: do not use this call on a device across cudaDeviceReset.
 */
pdssm_status pdssm_scan_fwd_noalloc(const pdssm_dims *dims,
                                    const int32_t *pi_dict,
                                    int64_t pi_head_stride, const int32_t *k,
                                    const void *d, const void *b,
                                    const void *c, pdssm_dtype in_dtype,
                                    const float *h0, float *y, float *h_last,
                                    int64_t chunk, void *stream);

/* Size in bytes of the static scratch array of pdssm_scan_fwd_noalloc. */
size_t pdssm_noalloc_scratch_bytes(void);

/*
 * pdssm_ws_status for the static scratch of pdssm_scan_fwd_noalloc on the
 * current device: synchronises the stream, returns what the kernels recorded
 * (PDSSM_ERR_BAD_INDEX, PDSSM_ERR_TIMEOUT) and clears it.  Allocates nothing.
 */
pdssm_status pdssm_noalloc_status(void *stream);

/*
 * Phase A alone, exposing each chunk's closed PD transfer (for tests of the
 * composed index maps, which must match bit for bit):
 *     h_e = P_{Pi_c} diag(Delta_c) h_{s-1} + v_c   for the chunk s..e.
 * Pi_out int32, Delta_out and v_out fp32, each [B][H][ceil(L/chunk)][N],
 * device.  ws as for pdssm_scan_fwd (for_bwd = 0).
 */
pdssm_status pdssm_chunk_transfers(const pdssm_dims *dims,
                                   const int32_t *pi_dict,
                                   int64_t pi_head_stride, const int32_t *k,
                                   const void *d, const void *b,
                                   pdssm_dtype in_dtype, int64_t chunk,
                                   int32_t *Pi_out, float *Delta_out,
                                   float *v_out, void *ws, size_t ws_bytes,
                                   void *stream);

/*
 * Test hook: copies the chunk transfers (Pi_c, Delta_c, v_c) and the carries
 * H_c = h_{e_c} (state at the end of chunk c) that the last pdssm_scan_fwd
 * left in `ws` (same dims, pi_head_stride and chunk), each
 * [B][H][ceil(L/chunk)][N] on the device; Pi_out int32, the others fp32.
 * Asynchronous on the stream.
 */
pdssm_status pdssm_ws_transfers(const pdssm_dims *dims, int64_t pi_head_stride,
                                int64_t chunk, const void *ws, size_t ws_bytes,
                                int32_t *Pi_out, float *Delta_out,
                                float *v_out, float *H_out, void *stream);

/*
 * Self-test of the kernels' bounded waits, with a failure made on purpose
 * but no fault: which = 0 runs the single-pass forward's look-back for a
 * chunk whose predecessor never publishes; which = 1 waits on an mbarrier
 * that nothing completes.  Each wait gives up after cap_ns (1 .. 2e9) of the
 * GPU's global timer and records PDSSM_ERR_TIMEOUT in the status word of
 * `ws` (at least pdssm_wait_selftest_ws_bytes() bytes, 256-byte aligned),
 * which pdssm_ws_status then returns.  The kernels' own waits use a cap of
 * 2 s.
 */
pdssm_status pdssm_wait_selftest(int which, int64_t cap_ns, void *ws,
                                 size_t ws_bytes, void *stream);
size_t pdssm_wait_selftest_ws_bytes(void);

/*
 * Checks every dictionary entry lies in [0, N) and every k in [0, K) on the
 * device, then synchronises the stream.  Returns PDSSM_ERR_BAD_INDEX if any
 * does not.  Uses the first 256 bytes of ws (ws_bytes >= 256).
 */
pdssm_status pdssm_validate(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k,
                            void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronises the stream, reads the workspace status word written by the
 * kernels (PDSSM_ERR_BAD_INDEX for a clamped index, PDSSM_ERR_TIMEOUT for a
 * staging wait that gave up) and clears it.  PDSSM_OK when nothing was
 * recorded.
 */
pdssm_status pdssm_ws_status(void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PDSSM_H */
