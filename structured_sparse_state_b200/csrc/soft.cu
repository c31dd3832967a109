// The dictionary from dense matrices, and the original PD-SSM's soft
// selection as a dense comparison path (Flash PD-SSM technical summary,
// Methodology §1):
//   * k_dict_hardmax   pi_k(j) = first argmax_i A_k[i][j]: the K column
//                      one-hot selectors Flash PD-SSM keeps as its dictionary;
//   * k_soft_maps      the original per-step transition: soft weights
//                      s = softmax(W u_t / tau) of the K scores, the dense
//                      combination M_t = sum_k s_k A_k (N x N per step), and
//                      its column hardmax -- the O(L N^2 K) generation that
//                      hard selection removes;
//   * k_scan_maps      the forward scan with one map per step.
// The maps are integer decisions taken by floating point, so the kernels
// follow a fixed fp32 arithmetic step by step (the logits' fma chain, the
// soft weights, the fma-chained mixture), which makes them reproducible bit
// for bit on any IEEE machine with a fused multiply-add.
#include "common.cuh"
#include "transfer_ops.cuh"

namespace pdssm {

// ---------------------------------------------------------------------------
// column hardmax
// ---------------------------------------------------------------------------
__global__ void k_dict_hardmax(int64_t n_mats, int N, const float *__restrict__ A,
                               int32_t *__restrict__ pi) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_mats * N) return;
    const int64_t m = idx / N;
    const int j = (int)(idx - m * N);
    const float *col = A + m * N * N + j;
    float best = __ldg(col);
    int bi = 0;
    for (int i = 1; i < N; ++i) {
        const float v = __ldg(col + (int64_t)i * N);
        if (v > best) {
            best = v;
            bi = i;
        }
    }
    pi[idx] = bi;
}

// ---------------------------------------------------------------------------
// soft selection
// ---------------------------------------------------------------------------

// exp(x) for x <= 0 by a published method, step by step in fp32: Cody-Waite
// reduction x = n ln2 + r with ln2 split in two parts, e^r by its Taylor
// series to degree 7 in Horner form with fused multiply-adds, times 2^n from
// its exponent bits; 0 below x = -86 (results stay normal).  The explicit
// _rn operations keep the compiler from contracting anything.
__device__ __forceinline__ float soft_exp(float x) {
    if (x < -86.0f) return 0.0f;
    const float n = rintf(__fmul_rn(x, 1.44269504f));
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
    const float two_n = __int_as_float(((int)n + 127) << 23);
    return __fmul_rn(p, two_n);
}

constexpr int kSoftSteps = 16;     // steps per CTA
constexpr int kSoftGroup = 4;      // steps per thread in the mixture
constexpr int kSoftThreads = 256;

struct SoftParams {
    const void *u;
    int u_bf16;
    const float *W;
    const float *A;
    int64_t a_hs;
    int32_t *maps;
    int64_t B, H, L;
    int D, K, N;
    float inv_tau;
};

// One CTA: kSoftSteps steps of one (b, h).  Threads (t, k) evaluate the
// logits as the fp32 fma chain in ascending q; one thread per step forms the
// soft weights; then each thread takes one column j for kSoftGroup steps and
// walks the rows i, mixing the K matrices with acc = fmaf(s_k, A_k[i][j],
// acc) in ascending k and keeping the first largest row.
__global__ void __launch_bounds__(kSoftThreads) k_soft_maps(const SoftParams p) {
    __shared__ float s_w[kSoftSteps][33];
    const int64_t tiles = (p.L + kSoftSteps - 1) / kSoftSteps;
    const int64_t bh = blockIdx.x / tiles;
    const int64_t t0 = (blockIdx.x - bh * tiles) * kSoftSteps;
    const int64_t bb = bh / p.H, h = bh - bb * p.H;
    const int nst = (int)imin64(kSoftSteps, p.L - t0);
    const int K = p.K, D = p.D, N = p.N;
    // logits
    for (int e = threadIdx.x; e < kSoftSteps * K; e += blockDim.x) {
        const int ts = e / K, kk = e - ts * K;
        if (ts >= nst) continue;
        const int64_t row = bb * p.L + t0 + ts;
        const float *wr = p.W + (h * K + kk) * D;
        float acc = 0.f;
        if (p.u_bf16) {
            const __nv_bfloat16 *ur = reinterpret_cast<const __nv_bfloat16 *>(p.u) + row * D;
            for (int q = 0; q < D; ++q) acc = fmaf(__ldg(wr + q), __bfloat162float(ur[q]), acc);
        } else {
            const float *ur = reinterpret_cast<const float *>(p.u) + row * D;
            for (int q = 0; q < D; ++q) acc = fmaf(__ldg(wr + q), __ldg(ur + q), acc);
        }
        s_w[ts][kk] = acc;
    }
    __syncthreads();
    // soft weights: m = max, e_k = exp((l_k - m) / tau), s_k = e_k / sum
    if (threadIdx.x < nst) {
        float *w = s_w[threadIdx.x];
        float m = w[0];
        for (int kk = 1; kk < K; ++kk)
            if (w[kk] > m) m = w[kk];
        float Z = 0.f;
        for (int kk = 0; kk < K; ++kk) {
            w[kk] = soft_exp(__fmul_rn(__fsub_rn(w[kk], m), p.inv_tau));
            Z = __fadd_rn(Z, w[kk]);
        }
        for (int kk = 0; kk < K; ++kk) w[kk] = __fdiv_rn(w[kk], Z);
    }
    __syncthreads();
    // mixture and column hardmax
    const float *Ah = p.A + h * p.a_hs;
    const int ngroups = kSoftSteps / kSoftGroup;
    for (int e = threadIdx.x; e < N * ngroups; e += blockDim.x) {
        const int j = e % N, g = e / N;
        const int tb = g * kSoftGroup;
        if (tb >= nst) continue;
        float best[kSoftGroup];
        int bi[kSoftGroup];
#pragma unroll
        for (int r = 0; r < kSoftGroup; ++r) {
            best[r] = 0.f;
            bi[r] = 0;
        }
        for (int i = 0; i < N; ++i) {
            float acc[kSoftGroup];
#pragma unroll
            for (int r = 0; r < kSoftGroup; ++r) acc[r] = 0.f;
            for (int kk = 0; kk < K; ++kk) {
                const float a = __ldg(Ah + (int64_t)kk * N * N + (int64_t)i * N + j);
#pragma unroll
                for (int r = 0; r < kSoftGroup; ++r) acc[r] = fmaf(s_w[tb + r][kk], a, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < kSoftGroup; ++r)
                if (i == 0 || acc[r] > best[r]) {
                    best[r] = acc[r];
                    bi[r] = i;
                }
        }
#pragma unroll
        for (int r = 0; r < kSoftGroup; ++r)
            if (tb + r < nst) p.maps[((bh * p.L) + t0 + tb + r) * N + j] = bi[r];
    }
}

// ---------------------------------------------------------------------------
// forward scan with one map per step: one warp per (b, h), sequential in t,
// the arbitrary-fan-in warp scatter of transfer_ops.cuh for every step
// ---------------------------------------------------------------------------
constexpr int kMapsWarps = 4;

template <typename T>
__global__ void __launch_bounds__(kMapsWarps * 32)
    k_scan_maps(int64_t BH, int64_t L, int N, const int32_t *__restrict__ maps,
                const T *__restrict__ d, const T *__restrict__ b, const T *__restrict__ c,
                const float *__restrict__ h0, float *__restrict__ y, float *__restrict__ h_last) {
    __shared__ ScatterScratch scr[kMapsWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t bh = (int64_t)blockIdx.x * kMapsWarps + warp;
    if (bh >= BH) return;
    ScatterScratch &sc = scr[warp];
    float h[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        h[r] = (h0 && e < N) ? h0[bh * N + e] : 0.f;
    }
    for (int64_t t = 0; t < L; ++t) {
        const int64_t row = (bh * L + t) * N;
        int P[2];
        float z[2], V[2], cv[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            if (e < N) {
                P[r] = __ldg(maps + row + e);
                z[r] = to_f<T>(d[row + e]) * h[r];
                V[r] = to_f<T>(b[row + e]);
                cv[r] = to_f<T>(c[row + e]);
            } else {
                P[r] = kPadIdx;
                z[r] = 0.f;
                V[r] = 0.f;
                cv[r] = 0.f;
            }
        }
        warp_scatter(P, z, V, h, sc, lane, false);
        float acc = fmaf(cv[1], h[1], cv[0] * h[0]);
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (lane == 0) y[bh * L + t] = acc;
    }
    if (h_last) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            if (e < N) h_last[bh * N + e] = h[r];
        }
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_dict_hardmax(int64_t n_mats, int N, const float *A, int32_t *pi,
                                cudaStream_t st) {
    const int64_t n = n_mats * N;
    if (n == 0) return cudaSuccess;
    k_dict_hardmax<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(n_mats, N, A, pi);
    return cudaGetLastError();
}

cudaError_t launch_soft_maps(const pdssm_dims &dm, const void *u, pdssm_dtype ut,
                             const float *W, const float *A, int64_t a_hs, float inv_tau,
                             int32_t *maps, cudaStream_t st) {
    SoftParams p;
    p.u = u;
    p.u_bf16 = ut == PDSSM_BF16;
    p.W = W;
    p.A = A;
    p.a_hs = a_hs;
    p.maps = maps;
    p.B = dm.B;
    p.H = dm.H;
    p.L = dm.L;
    p.D = (int)dm.D_in;
    p.K = (int)dm.K;
    p.N = (int)dm.N;
    p.inv_tau = inv_tau;
    const int64_t tiles = (dm.L + kSoftSteps - 1) / kSoftSteps;
    const int64_t grid = dm.B * dm.H * tiles;
    if (grid == 0) return cudaSuccess;
    k_soft_maps<<<(unsigned)grid, kSoftThreads, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_scan_maps(const pdssm_dims &dm, const int32_t *maps, const void *d,
                             const void *b, const void *c, pdssm_dtype dt, const float *h0,
                             float *y, float *h_last, cudaStream_t st) {
    const int64_t BH = dm.B * dm.H;
    const unsigned grid = (unsigned)((BH + kMapsWarps - 1) / kMapsWarps);
    if (dt == PDSSM_BF16)
        k_scan_maps<__nv_bfloat16><<<grid, kMapsWarps * 32, 0, st>>>(
            BH, dm.L, (int)dm.N, maps, reinterpret_cast<const __nv_bfloat16 *>(d),
            reinterpret_cast<const __nv_bfloat16 *>(b), reinterpret_cast<const __nv_bfloat16 *>(c),
            h0, y, h_last);
    else
        k_scan_maps<float><<<grid, kMapsWarps * 32, 0, st>>>(
            BH, dm.L, (int)dm.N, maps, reinterpret_cast<const float *>(d),
            reinterpret_cast<const float *>(b), reinterpret_cast<const float *>(c), h0, y, h_last);
    return cudaGetLastError();
}

}  // namespace pdssm
