// Forward chunked PD scan (Flash PD-SSM technical summary, Methodology §3):
//   phase A  chunk-local recurrence from a zero state: local readout, and the
//            chunk's closed PD transfer (Pi_c, Delta_c, v_c);
//   phase B  carry prefix scan over chunks: H_c = P_{Pi_c} diag(Delta_c) H_{c-1} + v_c;
//   phase C  carry correction of the readout.
//
// Phase C never rebuilds the state.  By linearity
//   h_t = v_t + P_{Pi_{s..t}} diag(Delta_{s..t}) H_{c-1},
// so y_t = <c_t, v_t> + sum_j c_t[pos_t(j)] * w_t(j), where each carry
// coordinate j travels one path pos_t(j) = pi_{k_t}(pos_{t-1}(j)) with weight
// w_t(j) = w_{t-1}(j) * d_t[pos_{t-1}(j)], w_{s-1}(j) = H_{c-1}[j].
// Phase A stores <c_t, v_t> in y; phase C adds the path sums.  Every
// correction term is a product (no cancellation, no division), which keeps
// the stiff regime (d down to 1e-4, products underflowing to 0) exact.
//
// The dictionary and its slot tables live in shared memory (one copy per CTA
// when all heads share it, one per warp otherwise); the state update is the
// deterministic slot gather pd_gather_step.
#include "common.cuh"

namespace pdssm {

// ---------------------------------------------------------------------------
// phase A
// ---------------------------------------------------------------------------
template <typename T, int NPL, bool FULL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_phaseA(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_a[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_a, warp, lane);
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int N = (int)p.N, K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);
    const bool with_y = p.y != nullptr;
    const int nt = with_y ? 3 : 2;

    const int rowb = N * (int)sizeof(T);
    unsigned char *wbase = sm_a + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    Ring<3> ring;
    ring.buf = wbase;
    ring.rowb = rowb;
    ring.esz = (int)sizeof(T);
    ring.tens_bytes = kTS * rowb;
    ring.stage_bytes = 3 * ring.tens_bytes;
    ring.ns = p.ns;
    ring.bulk = p.bulk != 0;
    float *pbuf = reinterpret_cast<float *>(wbase + p.ns * ring.stage_bytes);
    float *ybuf = pbuf + 2 * kPbStride;
    ring.bar0 = smem_u32(ybuf + kYbufFloats);
    const int64_t seq_row0 = bh * p.L;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + seq_row0 * rowb;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.b) + seq_row0 * rowb;
    ring.src[2] = with_y ? reinterpret_cast<const unsigned char *>(p.c) + seq_row0 * rowb
                         : ring.src[1];
    ring_init_bars(ring.bar0, p.ns, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    for (int i = 0; i < p.ns && i < ntiles; ++i)
        ring.issue(i, s + (int64_t)i * kTS, min(kTS, len - i * kTS), nt, lane);
    for (int i = p.ns; i < p.ns + kPrefetchTiles && i < ntiles; ++i)
        ring.prefetch(s + (int64_t)i * kTS, min(kTS, len - i * kTS), nt, lane);
    clear_pb(pbuf, lane);

    float h[NPL], Dl[NPL];
    int pos[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        h[r] = 0.f;
        Dl[r] = 1.f;
        pos[r] = min(lane * NPL + r, N - 1);
    }
    const int32_t *kp = p.k + bh * p.L + s;
    int kreg = load_k(kp, lane, lane < kTS && lane < len, K, p.status);

    for (int i = 0; i < ntiles; ++i) {
        const int stage = i % p.ns;
        if (!ring.wait(stage, (uint32_t)((i / p.ns) & 1))) {
            ring_abort(ring, i, min(ntiles, i + p.ns), p.status, lane);
            return;
        }
        const int t0 = i * kTS;
        const int n = min(kTS, len - t0);
        const int knext = load_k_raw(kp, t0 + kTS + lane, lane < kTS && t0 + kTS + lane < len);
        const T *rd = reinterpret_cast<const T *>(ring.tile(stage, 0));
        const T *rb = reinterpret_cast<const T *>(ring.tile(stage, 1));
        const T *rc = reinterpret_cast<const T *>(ring.tile(stage, 2));
#pragma unroll 2
        for (int q = 0; q < n; ++q, rd += N, rb += N, rc += N) {
            const int kk = __shfl_sync(kFull, kreg, q);
            const int *pk = sd.map + kk * N;
            float dv[NPL], bv[NPL];
            ld_own<T, NPL, FULL>(rd, lane, N, dv);
            ld_own<T, NPL, FULL>(rb, lane, N, bv);
            // transfer tracking: Delta picks up d at the column's current
            // position, then the selected map moves the column
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                if (FULL || lane * NPL + r < N) {
                    Dl[r] *= to_f<T>(rd[pos[r]]);
                    pos[r] = pk[pos[r]];
                }
            }
            pd_gather_step<NPL, FULL>(h, dv, bv, pbuf + (q & 1) * kPbStride,
                                      sd.tab + kk * (kDcap * 64) + lane * NPL, sd.fan[kk], pk,
                                      lane, N);
            if (with_y) {
                float cv[NPL];
                ld_own<T, NPL, FULL>(rc, lane, N, cv);
                float acc = cv[0] * h[0];
#pragma unroll
                for (int r = 1; r < NPL; ++r) acc = fmaf(cv[r], h[r], acc);
                ybuf[q * 33 + lane] = acc;
            }
        }
        __syncwarp();
        if (with_y) {
            const float ys = ybuf_row_sum(ybuf, lane, n);
            if (lane < n) p.y[bh * p.L + s + t0 + lane] = ys;
        }
        __syncwarp();
        if (i + p.ns < ntiles)
            ring.issue(stage, s + (int64_t)(i + p.ns) * kTS, min(kTS, len - (i + p.ns) * kTS), nt,
                       lane);
        {
            const int pf = i + p.ns + kPrefetchTiles;
            if (pf < ntiles) ring.prefetch(s + (int64_t)pf * kTS, min(kTS, len - pf * kTS), nt, lane);
        }
        kreg = clamp_k(knext, K, p.status);
    }
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        if (e < N) {
            p.Pi[o + e] = pos[r];
            p.Dl[o + e] = Dl[r];
            p.v[o + e] = h[r];
        }
    }
}

// ---------------------------------------------------------------------------
// phase C (carry correction in path form)
// ---------------------------------------------------------------------------
template <typename T, int NPL, bool FULL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_phaseC(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_c[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_c, warp, lane);
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int N = (int)p.N, K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    if (cidx == 0 && p.h0 == nullptr) return;   // zero initial state: nothing to correct
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    const int rowb = N * (int)sizeof(T);
    unsigned char *wbase = sm_c + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    Ring<2> ring;
    ring.buf = wbase;
    ring.rowb = rowb;
    ring.esz = (int)sizeof(T);
    ring.tens_bytes = kTS * rowb;
    ring.stage_bytes = 2 * ring.tens_bytes;
    ring.ns = p.ns;
    ring.bulk = p.bulk != 0;
    float *ybuf = reinterpret_cast<float *>(wbase + p.ns * ring.stage_bytes) + 2 * kPbStride;
    ring.bar0 = smem_u32(ybuf + kYbufFloats);
    const int64_t seq_row0 = bh * p.L;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + seq_row0 * rowb;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.c) + seq_row0 * rowb;
    ring_init_bars(ring.bar0, p.ns, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    for (int i = 0; i < p.ns && i < ntiles; ++i)
        ring.issue(i, s + (int64_t)i * kTS, min(kTS, len - i * kTS), 2, lane);
    for (int i = p.ns; i < p.ns + kPrefetchTiles && i < ntiles; ++i)
        ring.prefetch(s + (int64_t)i * kTS, min(kTS, len - i * kTS), 2, lane);

    float w[NPL];
    int pos[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        pos[r] = min(e, N - 1);
        w[r] = 0.f;
        if (e < N) w[r] = cidx == 0 ? p.h0[bh * p.N + e] : p.Hc[(unit - 1) * p.N + e];
    }
    const int32_t *kp = p.k + bh * p.L + s;
    float *yp = p.y + bh * p.L + s;
    int kreg = load_k(kp, lane, lane < kTS && lane < len, K, p.status);

    for (int i = 0; i < ntiles; ++i) {
        const int stage = i % p.ns;
        if (!ring.wait(stage, (uint32_t)((i / p.ns) & 1))) {
            ring_abort(ring, i, min(ntiles, i + p.ns), p.status, lane);
            return;
        }
        const int t0 = i * kTS;
        const int n = min(kTS, len - t0);
        const int knext = load_k_raw(kp, t0 + kTS + lane, lane < kTS && t0 + kTS + lane < len);
        const float yold = lane < n ? yp[t0 + lane] : 0.f;
        const T *rd = reinterpret_cast<const T *>(ring.tile(stage, 0));
        const T *rc = reinterpret_cast<const T *>(ring.tile(stage, 1));
#pragma unroll 2
        for (int q = 0; q < n; ++q, rd += N, rc += N) {
            const int kk = __shfl_sync(kFull, kreg, q);
            const int *pk = sd.map + kk * N;
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                if (FULL || lane * NPL + r < N) {
                    w[r] *= to_f<T>(rd[pos[r]]);
                    pos[r] = pk[pos[r]];
                    acc = fmaf(to_f<T>(rc[pos[r]]), w[r], acc);
                }
            }
            ybuf[q * 33 + lane] = acc;
        }
        __syncwarp();
        const float ys = ybuf_row_sum(ybuf, lane, n);
        if (lane < n) yp[t0 + lane] = yold + ys;
        __syncwarp();
        if (i + p.ns < ntiles)
            ring.issue(stage, s + (int64_t)(i + p.ns) * kTS, min(kTS, len - (i + p.ns) * kTS), 2,
                       lane);
        {
            const int pf = i + p.ns + kPrefetchTiles;
            if (pf < ntiles) ring.prefetch(s + (int64_t)pf * kTS, min(kTS, len - pf * kTS), 2, lane);
        }
        kreg = clamp_k(knext, K, p.status);
    }
}

// ---------------------------------------------------------------------------
// phase B: one CTA of nw warps per (b, h).  Chunks are split into nw
// contiguous segments: (1) each warp composes its segment's transfers,
// (2) warp 0 chains the segment aggregates from h0, (3) each warp re-applies
// its segment's transfers from its segment carry and stores every H_c.
// ---------------------------------------------------------------------------

// out = P_P diag(D) x + V for an arbitrary (composed) index map P: every
// lane scans all N sources in ascending j (maps composed over a chunk often
// collapse onto a few targets, so no bounded fan-in can be assumed).
// sP, sZ are this warp's scratch rows.  x and out may alias.
template <int NPL>
__device__ __forceinline__ void apply_scatter(const int (&P)[NPL], const float (&D)[NPL],
                                              const float (&V)[NPL], const float (&x)[NPL],
                                              float (&out)[NPL], int *sP, float *sZ, int N,
                                              int lane) {
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        if (e < N) {
            sP[e] = P[r];
            sZ[e] = D[r] * x[r];
        }
    }
    __syncwarp();
    float acc[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) acc[r] = 0.f;
#pragma unroll 4
    for (int j = 0; j < N; ++j) {
        const int pj = sP[j];
        const float zj = sZ[j];
#pragma unroll
        for (int r = 0; r < NPL; ++r)
            if (pj == lane * NPL + r) acc[r] += zj;
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < NPL; ++r) out[r] = lane * NPL + r < N ? acc[r] + V[r] : 0.f;
}

template <int NPL>
__device__ __forceinline__ void load_transfer(const ChunkParams &p, int64_t unit, int lane,
                                              int (&P)[NPL], float (&D)[NPL], float (&V)[NPL]) {
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        if (e < p.N) {
            P[r] = p.Pi[o + e];
            D[r] = p.Dl[o + e];
            V[r] = p.v[o + e];
        } else {
            P[r] = 0;
            D[r] = 0.f;
            V[r] = 0.f;
        }
    }
}

template <int NPL>
__global__ void k_phaseB(const ChunkParams p) {
    extern __shared__ __align__(16) unsigned char sm_b[];
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = (int)p.N;
    const int64_t bh = blockIdx.x;
    const int64_t C = p.C;
    int *sPall = reinterpret_cast<int *>(sm_b);                    // [nw][64]
    float *sZall = reinterpret_cast<float *>(sPall + nw * kMaxN);  // [nw][64]
    float *sDall = sZall + nw * kMaxN;                             // [nw][64]
    int *aggP = reinterpret_cast<int *>(sDall + nw * kMaxN);       // [nw][64]
    float *aggD = reinterpret_cast<float *>(aggP + nw * kMaxN);
    float *aggV = aggD + nw * kMaxN;
    float *carry = aggV + nw * kMaxN;                              // [nw][64]
    int *sP = sPall + warp * kMaxN;
    float *sZ = sZall + warp * kMaxN;
    float *sD = sDall + warp * kMaxN;

    const int64_t c0 = C * warp / nw, c1 = C * (warp + 1) / nw;
    const int64_t u0 = bh * C;

    // (1) segment aggregate: T_{c1-1} o ... o T_{c0}
    if (c0 < c1) {
        int aP[NPL];
        float aD[NPL], aV[NPL];
        load_transfer<NPL>(p, u0 + c0, lane, aP, aD, aV);
        int P2[NPL];
        float D2[NPL], V2[NPL];
        if (c0 + 1 < c1) load_transfer<NPL>(p, u0 + c0 + 1, lane, P2, D2, V2);
        for (int64_t c = c0 + 1; c < c1; ++c) {
            int Pn[NPL];
            float Dn[NPL], Vn[NPL];
            if (c + 1 < c1) load_transfer<NPL>(p, u0 + c + 1, lane, Pn, Dn, Vn);
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                if (e < N) {
                    sP[e] = P2[r];
                    sD[e] = D2[r];
                }
            }
            __syncwarp();
            int nP[NPL];
            float nD[NPL];
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                nP[r] = sP[aP[r]];
                nD[r] = aD[r] * sD[aP[r]];
            }
            __syncwarp();
            apply_scatter<NPL>(P2, D2, V2, aV, aV, sP, sZ, N, lane);
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                aP[r] = nP[r];
                aD[r] = nD[r];
                if (c + 1 < c1) {
                    P2[r] = Pn[r];
                    D2[r] = Dn[r];
                    V2[r] = Vn[r];
                }
            }
        }
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            if (e < N) {
                aggP[warp * kMaxN + e] = aP[r];
                aggD[warp * kMaxN + e] = aD[r];
                aggV[warp * kMaxN + e] = aV[r];
            }
        }
    }
    __syncthreads();
    // (2) chain the segment aggregates
    if (warp == 0) {
        float S[NPL];
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            S[r] = (e < N && p.h0) ? p.h0[bh * p.N + e] : 0.f;
        }
        for (int w = 0; w < nw; ++w) {
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                if (e < N) carry[w * kMaxN + e] = S[r];
            }
            if (C * w / nw < C * (w + 1) / nw) {
                int P[NPL];
                float D[NPL], V[NPL];
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    const int e = lane * NPL + r;
                    P[r] = e < N ? aggP[w * kMaxN + e] : 0;
                    D[r] = e < N ? aggD[w * kMaxN + e] : 0.f;
                    V[r] = e < N ? aggV[w * kMaxN + e] : 0.f;
                }
                apply_scatter<NPL>(P, D, V, S, S, sP, sZ, N, lane);
            }
        }
        if (p.h_last) {
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                if (e < N) p.h_last[bh * p.N + e] = S[r];
            }
        }
    }
    __syncthreads();
    // (3) fill the carries of this warp's segment
    float x[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        x[r] = e < N ? carry[warp * kMaxN + e] : 0.f;
    }
    if (c0 < c1) {
        int P[NPL];
        float D[NPL], V[NPL];
        load_transfer<NPL>(p, u0 + c0, lane, P, D, V);
        for (int64_t c = c0; c < c1; ++c) {
            int Pn[NPL];
            float Dn[NPL], Vn[NPL];
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                Pn[r] = 0;
                Dn[r] = 0.f;
                Vn[r] = 0.f;
            }
            if (c + 1 < c1) load_transfer<NPL>(p, u0 + c + 1, lane, Pn, Dn, Vn);
            apply_scatter<NPL>(P, D, V, x, x, sP, sZ, N, lane);
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                if (e < N) p.Hc[(u0 + c) * p.N + e] = x[r];
                P[r] = Pn[r];
                D[r] = Dn[r];
                V[r] = Vn[r];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <typename KernT>
static cudaError_t launch_chunk(KernT kern, const ChunkParams &p, size_t, cudaStream_t st) {
    return launch_units(kern, p, p.smem_per_warp, st);
}

// Template choice: NPL = elements per lane, FULL = the state fills the warp.
#define PDSSM_DISPATCH(KERNEL, p, st, smem)                                       \
    do {                                                                         \
        if ((p).N == 64) return launch_chunk(KERNEL<T, 2, true>, p, smem, st);   \
        if ((p).N > 32) return launch_chunk(KERNEL<T, 2, false>, p, smem, st);   \
        if ((p).N == 32) return launch_chunk(KERNEL<T, 1, true>, p, smem, st);   \
        return launch_chunk(KERNEL<T, 1, false>, p, smem, st);                   \
    } while (0)

template <typename T>
static cudaError_t phaseA_t(ChunkParams p, cudaStream_t st) {
    const int rowb = (int)p.N * (int)sizeof(T);
    p.smem_per_warp = warp_smem_bytes(p.ns, 3, rowb);
    const size_t smem = 0;
    PDSSM_DISPATCH(k_phaseA, p, st, smem);
}

template <typename T>
static cudaError_t phaseC_t(ChunkParams p, cudaStream_t st) {
    const int rowb = (int)p.N * (int)sizeof(T);
    p.smem_per_warp = warp_smem_bytes(p.ns, 2, rowb);
    const size_t smem = 0;
    PDSSM_DISPATCH(k_phaseC, p, st, smem);
}

cudaError_t launch_phaseA(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st) {
    if (p.units == 0) return cudaSuccess;
    if (fast_path(p)) return launch_phaseA_fast(p, dt, st);
    return dt == PDSSM_BF16 ? phaseA_t<__nv_bfloat16>(p, st) : phaseA_t<float>(p, st);
}

cudaError_t launch_phaseC(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st) {
    if (p.units == 0) return cudaSuccess;
    if (fast_path(p)) return launch_phaseC_fast(p, dt, st);
    return dt == PDSSM_BF16 ? phaseC_t<__nv_bfloat16>(p, st) : phaseC_t<float>(p, st);
}

cudaError_t launch_phaseB(const ChunkParams &p, cudaStream_t st) {
    if (p.units == 0) return cudaSuccess;
    const int nw = (int)imin64(32, p.C);
    const size_t smem = (size_t)nw * kMaxN * 4 * 7;
    const int64_t BH = p.B * p.H;
    cudaError_t e;
    if (p.N > 32) {
        e = cudaFuncSetAttribute(k_phaseB<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        k_phaseB<2><<<(unsigned)BH, nw * 32, smem, st>>>(p);
    } else {
        e = cudaFuncSetAttribute(k_phaseB<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        k_phaseB<1><<<(unsigned)BH, nw * 32, smem, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace pdssm
