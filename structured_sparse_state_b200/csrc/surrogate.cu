// Straight-through surrogate gradients of the hard selection and of the
// column-hardmax dictionary (Flash PD-SSM technical summary, Methodology §2:
// hard forward; in the backward the discrete choices are replaced by
// tempered softmaxes so that gradients reach the selection weights and the
// dense dictionary matrices).  Each choice is relaxed on its own around the
// hard trajectory (lambda_t = dl/dh_t from pdssm_scan_bwd, z_t = d_t h_{t-1}):
//   selection:  g_s[t,k] = sum_j lambda_t[pi_k(j)] z_t[j]        (K gathers)
//               g_l[t,k] = inv_tau_s s_k (g_s[t,k] - sum_k' s_k' g_s[t,k'])
//               g_W[h,k,:] = sum_{b,t} g_l[b,h,t,k] u[b,t,:]
//   dictionary: G_k = sum_{t : k_t = k} lambda_t z_t^T            (N^2 per step)
//               g_A[k][:,j] = inv_tau_a Q[:,j] (G[:,j] - <Q[:,j], G[:,j]>),
//               Q_k = column softmax of A_k * inv_tau_a.
// Kernels:
//   k_surr_steps   one warp per chunk: the hard state from the forward's
//                  carry, lambda, z, g_s, the soft weights, g_l; writes g_l
//                  and z_t;
//   k_surr_dict    CTA (matrix, slice): the outer products of the steps that
//                  selected the matrix, in a 64 x 64 register tile;
//   k_surr_wgrad   CTA (head, slice): g_l x u over the slice's rows;
//   k_surr_final   sums the slices in order and applies the column softmax.
// Every sum runs in a fixed order, so results are deterministic.
#include "common.cuh"
#include "transfer_ops.cuh"

namespace pdssm {

constexpr int kSurrWarps = 4;
constexpr int kSurrSlices = 32;      // slices of the step range per output block
constexpr int kSurrBatch = 16;       // rows staged together in the reductions

struct SurrParams {
    int64_t B, H, L, C, chunk;
    int N, K, D;
    int64_t a_hs;                    // head stride of A (0: shared)
    int Hd;                          // dictionaries: H if a_hs else 1
    const void *u;
    int u_bf16;
    const float *W;                  // [H][K][D]
    const float *A;                  // matrix (hd, k) at A + hd*a_hs + k*N*N
    const int32_t *pi;               // hard dictionary [Hd][K][N]
    const int32_t *k;                // [B][H][L]
    const void *d, *b;
    int in_bf16;
    const float *h0;                 // [B][H][N] or NULL
    const float *Hc;                 // carries [B*H][C][N] from the forward's workspace
    const float *lam;                // lambda = g_b [B][H][L][N]
    float inv_tau_s, inv_tau_a;
    float *g_l;                      // [B][H][L][K]
    float *z;                        // scratch [B][H][L][N]
    float *gA_part;                  // scratch [Hd*K][kSurrSlices][N][N]
    float *gW_part;                  // scratch [H][kSurrSlices][K][D]
    float *g_A;                      // [Hd][K][N][N]
    float *g_W;                      // [H][K][D]
};

template <typename T>
__device__ __forceinline__ float ld_elem(const void *base, int64_t idx) {
    return to_f<T>(reinterpret_cast<const T *>(base)[idx]);
}

// ---------------------------------------------------------------------------
// per-step quantities, one warp per chunk
// ---------------------------------------------------------------------------
// Per-warp shared memory of k_surr_steps (float offsets): W [K][D],
// pi [K][N] (ints), lam [64], red [K][33], u [D], then the scatter scratch.
struct SurrLayout {
    int W, pi, lam, red, u, sc, floats;
};
__host__ __device__ inline SurrLayout surr_layout(int K, int N, int D) {
    SurrLayout l;
    l.W = 0;
    l.pi = l.W + K * D;
    l.lam = l.pi + K * N;
    l.red = l.lam + 64;
    l.u = l.red + K * 33;
    l.sc = (l.u + D + 3) / 4 * 4;
    l.floats = l.sc + (int)(sizeof(ScatterScratch) / 4);
    return l;
}

template <typename T>
__global__ void __launch_bounds__(kSurrWarps * 32) k_surr_steps(const SurrParams p) {
    extern __shared__ __align__(16) float sm_surr[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = p.N, K = p.K, D = p.D;
    const SurrLayout lay = surr_layout(K, N, D);
    float *base = sm_surr + warp * lay.floats;
    float *sW = base + lay.W;
    int *spi = reinterpret_cast<int *>(base + lay.pi);
    float *slam = base + lay.lam;
    float *sred = base + lay.red;
    float *su = base + lay.u;
    ScatterScratch &sc = *reinterpret_cast<ScatterScratch *>(base + lay.sc);
    const int64_t unit = (int64_t)blockIdx.x * kSurrWarps + warp;
    if (unit >= p.B * p.H * p.C) return;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t bb = bh / p.H, hh = bh - bb * p.H;
    const int64_t hd = p.a_hs ? hh : 0;
    for (int i = lane; i < K * D; i += 32) sW[i] = p.W[hh * K * D + i];
    for (int i = lane; i < K * N; i += 32) spi[i] = p.pi[hd * K * N + i];
    // state entering the chunk: the forward's carry (lane l holds l, l + 32)
    float x[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        x[r] = e >= N ? 0.f
                      : cidx == 0 ? (p.h0 ? p.h0[bh * N + e] : 0.f)
                                  : p.Hc[(unit - 1) * N + e];
    }
    __syncwarp();
    const int64_t s0 = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s0);
    for (int q = 0; q < len; ++q) {
        const int64_t t = s0 + q;
        const int64_t row = bh * p.L + t;
        float z[2], bv[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            if (e < N) {
                z[r] = ld_elem<T>(p.d, row * N + e) * x[r];
                bv[r] = ld_elem<T>(p.b, row * N + e);
                slam[e] = p.lam[row * N + e];
                p.z[row * N + e] = z[r];
            } else {
                z[r] = 0.f;
                bv[r] = 0.f;
            }
        }
        for (int i = lane; i < D; i += 32)
            su[i] = p.u_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(
                                   p.u)[(bb * p.L + t) * D + i])
                             : reinterpret_cast<const float *>(p.u)[(bb * p.L + t) * D + i];
        __syncwarp();
        // g_s: this lane's columns' share for every map, then a transposed sum
        for (int kk = 0; kk < K; ++kk) {
            float part = 0.f;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int e = lane + 32 * r;
                if (e < N) part = fmaf(slam[spi[kk * N + e]], z[r], part);
            }
            sred[kk * 33 + lane] = part;
        }
        __syncwarp();
        float gs = 0.f, lg = -INFINITY;
        if (lane < K) {
            for (int i = 0; i < 32; ++i) gs += sred[lane * 33 + i];
            // the selection logit in the fp32 fma chain of pdssm_select
            float acc = 0.f;
            for (int qd = 0; qd < D; ++qd) acc = fmaf(sW[lane * D + qd], su[qd], acc);
            lg = acc;
        }
        // soft weights over the K lanes, and g_l
        float m = lg;
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
        const float e = lane < K ? expf((lg - m) * p.inv_tau_s) : 0.f;
        float Z = e;
#pragma unroll
        for (int o = 16; o; o >>= 1) Z += __shfl_xor_sync(kFull, Z, o);
        const float s = e / Z;
        float sg = s * gs;
#pragma unroll
        for (int o = 16; o; o >>= 1) sg += __shfl_xor_sync(kFull, sg, o);
        if (lane < K) p.g_l[row * K + lane] = p.inv_tau_s * s * (gs - sg);
        // the hard step to h_t (indices checked by the forward; clamped here)
        const int kt = min(max(__ldg(p.k + row), 0), K - 1);
        int P[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e2 = lane + 32 * r;
            P[r] = e2 < N ? spi[kt * N + e2] : kPadIdx;
        }
        warp_scatter(P, z, bv, x, sc, lane, false);
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// dictionary gradient: G_k partial sums over slices of the (b, h, t) rows
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_surr_dict(const SurrParams p) {
    __shared__ float s_lam[kSurrBatch][64];
    __shared__ float s_z[kSurrBatch][64];
    __shared__ int64_t s_list[256];
    __shared__ int s_wc[8];
    const int N = p.N, K = p.K;
    const int m = blockIdx.x;            // matrix (hd, k)
    const int slice = blockIdx.y;
    const int hd = m / K, kk = m - hd * K;
    const int64_t rows = p.B * p.H * p.L;
    const int64_t r0 = rows * slice / kSurrSlices, r1 = rows * (slice + 1) / kSurrSlices;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // thread (ti, tj): rows 4 ti .. 4 ti + 3, columns 4 tj .. 4 tj + 3 of G
    const int ti = threadIdx.x >> 4, tj = threadIdx.x & 15;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) acc[a][c2] = 0.f;
    for (int64_t base = r0; base < r1; base += 256) {
        // the rows of this block of 256 that selected matrix m, in order
        const int64_t r = base + threadIdx.x;
        bool hit = false;
        if (r < r1) {
            const int64_t h = (r / p.L) % p.H;
            hit = (p.a_hs == 0 || h == hd) && __ldg(p.k + r) == kk;
        }
        const unsigned bal = __ballot_sync(kFull, hit);
        if (lane == 0) s_wc[warp] = __popc(bal);
        __syncthreads();
        int before = 0, cnt = 0;
        for (int w = 0; w < 8; ++w) {
            before += w < warp ? s_wc[w] : 0;
            cnt += s_wc[w];
        }
        if (hit) s_list[before + __popc(bal & ((1u << lane) - 1u))] = r;
        __syncthreads();
        for (int q0 = 0; q0 < cnt; q0 += kSurrBatch) {
            const int nb = min(kSurrBatch, cnt - q0);
            for (int e = threadIdx.x; e < nb * 64; e += blockDim.x) {
                const int q = e >> 6, col = e & 63;
                const int64_t rr = s_list[q0 + q];
                s_lam[q][col] = col < N ? p.lam[rr * N + col] : 0.f;
                s_z[q][col] = col < N ? p.z[rr * N + col] : 0.f;
            }
            __syncthreads();
            for (int q = 0; q < nb; ++q) {
                float li[4], zj[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    li[a] = s_lam[q][4 * ti + a];
                    zj[a] = s_z[q][4 * tj + a];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) acc[a][c2] = fmaf(li[a], zj[c2], acc[a][c2]);
            }
            __syncthreads();
        }
    }
    float *out = p.gA_part + ((int64_t)m * kSurrSlices + slice) * N * N;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
            const int i = 4 * ti + a, j = 4 * tj + c2;
            if (i < N && j < N) out[i * N + j] = acc[a][c2];
        }
}

// ---------------------------------------------------------------------------
// weight gradient: g_W[h] partial sums over slices of the (b, t) rows
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_surr_wgrad(const SurrParams p) {
    __shared__ float s_g[kSurrBatch][32];
    __shared__ float s_u[kSurrBatch][256];
    const int K = p.K, D = p.D;
    const int64_t hh = blockIdx.x;
    const int slice = blockIdx.y;
    const int64_t rows = p.B * p.L;
    const int64_t r0 = rows * slice / kSurrSlices, r1 = rows * (slice + 1) / kSurrSlices;
    const int KD = K * D;
    constexpr int kPer = 32;             // outputs per thread (K*D <= 8192)
    float acc[kPer];
#pragma unroll
    for (int a = 0; a < kPer; ++a) acc[a] = 0.f;
    for (int64_t base = r0; base < r1; base += kSurrBatch) {
        const int cnt = (int)imin64(kSurrBatch, r1 - base);
        for (int e = threadIdx.x; e < cnt * 32; e += blockDim.x) {
            const int q = e >> 5, kk = e & 31;
            const int64_t r = base + q;
            const int64_t bb = r / p.L, t = r - bb * p.L;
            s_g[q][kk] = kk < K ? p.g_l[((bb * p.H + hh) * p.L + t) * K + kk] : 0.f;
        }
        for (int e = threadIdx.x; e < cnt * D; e += blockDim.x) {
            const int q = e / D, qd = e - q * D;
            const int64_t r = base + q;
            s_u[q][qd] = p.u_bf16 ? __bfloat162float(
                                        reinterpret_cast<const __nv_bfloat16 *>(p.u)[r * D + qd])
                                  : reinterpret_cast<const float *>(p.u)[r * D + qd];
        }
        __syncthreads();
        for (int q = 0; q < cnt; ++q) {
#pragma unroll
            for (int a = 0; a < kPer; ++a) {
                const int o = threadIdx.x + a * 256;
                if (o < KD) acc[a] = fmaf(s_g[q][o / D], s_u[q][o % D], acc[a]);
            }
        }
        __syncthreads();
    }
    float *out = p.gW_part + (hh * kSurrSlices + slice) * (int64_t)KD;
#pragma unroll
    for (int a = 0; a < kPer; ++a) {
        const int o = threadIdx.x + a * 256;
        if (o < KD) out[o] = acc[a];
    }
}

// ---------------------------------------------------------------------------
// sums over the slices (in order), and the column softmax of the dictionary
// ---------------------------------------------------------------------------
__global__ void k_surr_final_w(const SurrParams p) {
    const int64_t KD = (int64_t)p.K * p.D;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= p.H * KD) return;
    const int64_t hh = idx / KD, o = idx - hh * KD;
    float s = 0.f;
    for (int sl = 0; sl < kSurrSlices; ++sl) s += p.gW_part[(hh * kSurrSlices + sl) * KD + o];
    p.g_W[idx] = s;
}

// One thread per column j of matrix m: G[:, j] summed over the slices, the
// column softmax Q[:, j] of A * inv_tau_a, then g_A[:, j].
__global__ void k_surr_final_a(const SurrParams p) {
    const int N = p.N;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nm = (int64_t)p.Hd * p.K;
    if (idx >= nm * N) return;
    const int64_t m = idx / N;
    const int j = (int)(idx - m * N);
    const int64_t hd = m / p.K, kk = m - hd * p.K;
    const float *Am = p.A + hd * p.a_hs + kk * N * N;
    float mx = Am[j];
    for (int i = 1; i < N; ++i) mx = fmaxf(mx, Am[i * N + j]);
    float Z = 0.f;
    for (int i = 0; i < N; ++i) Z += expf((Am[i * N + j] - mx) * p.inv_tau_a);
    float dotq = 0.f;
    for (int i = 0; i < N; ++i) {
        float g = 0.f;
        for (int sl = 0; sl < kSurrSlices; ++sl)
            g += p.gA_part[(m * kSurrSlices + sl) * N * N + i * N + j];
        const float q = expf((Am[i * N + j] - mx) * p.inv_tau_a) / Z;
        dotq = fmaf(q, g, dotq);
        p.g_A[m * N * N + i * N + j] = g;   // G for now
    }
    for (int i = 0; i < N; ++i) {
        const float q = expf((Am[i * N + j] - mx) * p.inv_tau_a) / Z;
        const float g = p.g_A[m * N * N + i * N + j];
        p.g_A[m * N * N + i * N + j] = p.inv_tau_a * q * (g - dotq);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t surrogate_scratch_bytes(const pdssm_dims &dm, int64_t a_hs) {
    const int64_t Hd = a_hs ? dm.H : 1;
    const size_t z = align256((size_t)(dm.B * dm.H * dm.L * dm.N) * 4);
    const size_t ga = align256((size_t)(Hd * dm.K * kSurrSlices * dm.N * dm.N) * 4);
    const size_t gw = align256((size_t)(dm.H * kSurrSlices * dm.K * dm.D_in) * 4);
    return z + ga + gw;
}

cudaError_t launch_surrogate(const pdssm_dims &dm, const void *u, pdssm_dtype ut, const float *W,
                             const float *A, int64_t a_hs, const int32_t *pi, const int32_t *k,
                             const void *d, const void *b, pdssm_dtype dt, const float *h0,
                             const float *Hc, int64_t chunk, const float *lam, float inv_tau_s,
                             float inv_tau_a, void *scratch, float *g_l, float *g_W, float *g_A,
                             cudaStream_t st) {
    SurrParams p;
    p.B = dm.B;
    p.H = dm.H;
    p.L = dm.L;
    p.chunk = chunk;
    p.C = (dm.L + chunk - 1) / chunk;
    p.N = (int)dm.N;
    p.K = (int)dm.K;
    p.D = (int)dm.D_in;
    p.a_hs = a_hs;
    p.Hd = a_hs ? (int)dm.H : 1;
    p.u = u;
    p.u_bf16 = ut == PDSSM_BF16;
    p.W = W;
    p.A = A;
    p.pi = pi;
    p.k = k;
    p.d = d;
    p.b = b;
    p.in_bf16 = dt == PDSSM_BF16;
    p.h0 = h0;
    p.Hc = Hc;
    p.lam = lam;
    p.inv_tau_s = inv_tau_s;
    p.inv_tau_a = inv_tau_a;
    p.g_l = g_l;
    p.g_W = g_W;
    p.g_A = g_A;
    unsigned char *s = reinterpret_cast<unsigned char *>(scratch);
    const int64_t Hd = p.Hd;
    p.z = reinterpret_cast<float *>(s);
    s += align256((size_t)(dm.B * dm.H * dm.L * dm.N) * 4);
    p.gA_part = reinterpret_cast<float *>(s);
    s += align256((size_t)(Hd * dm.K * kSurrSlices * dm.N * dm.N) * 4);
    p.gW_part = reinterpret_cast<float *>(s);
    const int64_t units = dm.B * dm.H * p.C;
    if (units > 0) {
        const size_t smem =
            (size_t)kSurrWarps * surr_layout(p.K, p.N, p.D).floats * sizeof(float);
        auto kern = p.in_bf16 ? k_surr_steps<__nv_bfloat16> : k_surr_steps<float>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)((units + kSurrWarps - 1) / kSurrWarps), kSurrWarps * 32, smem, st>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    k_surr_dict<<<dim3((unsigned)(Hd * dm.K), kSurrSlices), 256, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_surr_wgrad<<<dim3((unsigned)dm.H, kSurrSlices), 256, 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t nw = dm.H * dm.K * dm.D_in;
    k_surr_final_w<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t na = Hd * dm.K * dm.N;
    k_surr_final_a<<<(unsigned)((na + 127) / 128), 128, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace pdssm
