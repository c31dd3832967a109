// Exact adjoint of the chunked PD scan (Breaking the Memory Wall / PGF,
// abstract and framework stages: chunk the sequence, evolve each chunk,
// take derivatives from the transfers, combine the chunks).
//
// With M_t = P_{k_t} diag(d_t) and lambda_t = dl/dh_t:
//   lambda_t = g_y[t] c_t + M_{t+1}^T lambda_{t+1},   (M^T x)[j] = d[j] x[pi(j)]
// -- a gather, so the reverse recurrence needs no scatter plan.
// Per chunk s..e the gradient leaving the chunk towards h_{s-1} is
//   Lambda_{c-1} = w_c + diag(Delta_c) P_{Pi_c}^T Lambda_c,
// i.e. Lambda_{c-1}[j] = w_c[j] + Delta_c[j] * Lambda_c[Pi_c[j]], with
// w_c = M_s^T lambda^loc_s from the chunk's own readouts.  The forward's
// (Pi_c, Delta_c) are reused; h inside a chunk is recomputed from H_{c-1}.
//   bwd phase A  w_c per chunk (reverse sweep from a zero carry)
//   bwd phase B  Lambda_c for every chunk and g_h0 = Lambda_{-1}
//   bwd phase C  recompute h, sweep back, emit g_b, g_c, g_d.
#include "common.cuh"

namespace pdssm {

// bwd phase C warp: ring, exchange buffers (2 x kPbStride), readout buffer,
// lambda buffers (2 x kPbStride), checkpoints (16 x 64), tile states (17 x 64)
constexpr int kBwdExtraFloats = 2 * kPbStride + (kBwdMaxChunk / kTS) * kMaxN + (kTS + 1) * kMaxN;
__host__ __device__ inline int bwd_warp_smem_bytes(int ns, int nt, int rowb) {
    return warp_smem_bytes(ns, nt, rowb, kBwdExtraFloats * 4);
}

template <int NPL, bool FULL>
__device__ __forceinline__ void st_own(float *row, int lane, int N, const float (&v)[NPL]) {
    if constexpr (FULL && NPL == 2) {
        *reinterpret_cast<float2 *>(row + 2 * lane) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            if (FULL || e < N) row[e] = v[r];
        }
    }
}

template <int NPL, bool FULL>
__device__ __forceinline__ void own_targets2(const int *pk, int lane, int N, int (&tgt)[NPL]) {
    if constexpr (FULL && NPL == 2) {
        const int2 q = *reinterpret_cast<const int2 *>(pk + 2 * lane);
        tgt[0] = q.x;
        tgt[1] = q.y;
    } else {
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            tgt[r] = (FULL || e < N) ? pk[e] : 0;
        }
    }
}

// ---------------------------------------------------------------------------
// bwd phase A: w_c = M_s^T lambda^loc_s with lambda^loc from a zero carry
// ---------------------------------------------------------------------------
template <typename T, int NPL, bool FULL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_bwdA(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_ba[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_ba, warp, lane);
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int N = (int)p.N, K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    unsigned char *wbase = sm_ba + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    const int rowb = N * (int)sizeof(T);
    Ring<2> ring;
    ring.buf = wbase;
    ring.rowb = rowb;
    ring.esz = (int)sizeof(T);
    ring.tens_bytes = kTS * rowb;
    ring.stage_bytes = 2 * ring.tens_bytes;
    ring.ns = p.ns;
    ring.bulk = p.bulk != 0;
    float *lbuf = reinterpret_cast<float *>(wbase + p.ns * ring.stage_bytes);
    ring.bar0 = smem_u32(lbuf + 2 * kPbStride + kYbufFloats);
    const int64_t seq_row0 = bh * p.L;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + seq_row0 * rowb;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.c) + seq_row0 * rowb;
    ring_init_bars(ring.bar0, p.ns, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    auto tile_of = [&](int j) { return ntiles - 1 - j; };   // reverse order
    for (int j = 0; j < p.ns && j < ntiles; ++j) {
        const int ti = tile_of(j);
        ring.issue(j, s + (int64_t)ti * kTS, min(kTS, len - ti * kTS), 2, lane);
    }
    for (int j = p.ns; j < p.ns + kPrefetchTiles && j < ntiles; ++j) {
        const int ti = tile_of(j);
        ring.prefetch(s + (int64_t)ti * kTS, min(kTS, len - ti * kTS), 2, lane);
    }
    const int32_t *kp = p.k + bh * p.L + s;
    const float *gyp = p.g_y + bh * p.L + s;
    float mu[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) mu[r] = 0.f;
    int t0 = (ntiles - 1) * kTS;
    int kreg = load_k(kp, t0 + lane, lane < kTS && t0 + lane < len, K, p.status);
    float gyreg = (lane < kTS && t0 + lane < len) ? gyp[t0 + lane] : 0.f;

    for (int j = 0; j < ntiles; ++j) {
        const int stage = j % p.ns;
        if (!ring.wait(stage, (uint32_t)((j / p.ns) & 1))) {
            ring_abort(ring, j, min(ntiles, j + p.ns), p.status, lane);
            return;
        }
        t0 = tile_of(j) * kTS;
        const int n = min(kTS, len - t0);
        const int tp = t0 - kTS;   // the tile processed next
        const bool vp = lane < kTS && tp >= 0;
        const int knext = load_k_raw(kp, tp + lane, vp);
        const float gynext = vp ? gyp[tp + lane] : 0.f;
        const T *td = reinterpret_cast<const T *>(ring.tile(stage, 0));
        const T *tc = reinterpret_cast<const T *>(ring.tile(stage, 1));
#pragma unroll 2
        for (int q = n - 1; q >= 0; --q) {
            const int kk = __shfl_sync(kFull, kreg, q);
            const float gy = __shfl_sync(kFull, gyreg, q);
            float dv[NPL], cv[NPL], lam[NPL];
            ld_own<T, NPL, FULL>(td + q * N, lane, N, dv);
            ld_own<T, NPL, FULL>(tc + q * N, lane, N, cv);
#pragma unroll
            for (int r = 0; r < NPL; ++r) lam[r] = gy * cv[r] + mu[r];
            float *lb = lbuf + (q & 1) * kPbStride;
            st_own<NPL, FULL>(lb, lane, N, lam);
            __syncwarp();
            int tgt[NPL];
            own_targets2<NPL, FULL>(sd.map + kk * N, lane, N, tgt);
#pragma unroll
            for (int r = 0; r < NPL; ++r) mu[r] = dv[r] * lb[tgt[r]];
        }
        __syncwarp();
        if (j + p.ns < ntiles) {
            const int tn = tile_of(j + p.ns);
            ring.issue(stage, s + (int64_t)tn * kTS, min(kTS, len - tn * kTS), 2, lane);
        }
        if (j + p.ns + kPrefetchTiles < ntiles) {
            const int tp2 = tile_of(j + p.ns + kPrefetchTiles);
            ring.prefetch(s + (int64_t)tp2 * kTS, min(kTS, len - tp2 * kTS), 2, lane);
        }
        kreg = clamp_k(knext, K, p.status);
        gyreg = gynext;
    }
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        if (e < N) p.wc[o + e] = mu[r];
    }
}

// ---------------------------------------------------------------------------
// bwd phase B: reverse carry scan.  R_c(x)[j] = w_c[j] + Delta_c[j] x[Pi_c[j]]
// maps Lambda_c to Lambda_{c-1}; compositions stay gathers:
//   (R_a o R_b): w = w_a + Delta_a * w_b[Pi_a], Delta = Delta_a * Delta_b[Pi_a],
//                Pi = Pi_b[Pi_a].
// ---------------------------------------------------------------------------
template <int NPL>
__device__ __forceinline__ void load_rev(const ChunkParams &p, int64_t unit, int lane,
                                         int (&P)[NPL], float (&D)[NPL], float (&W)[NPL]) {
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        if (e < p.N) {
            P[r] = p.Pi[o + e];
            D[r] = p.Dl[o + e];
            W[r] = p.wc[o + e];
        } else {
            P[r] = 0;
            D[r] = 0.f;
            W[r] = 0.f;
        }
    }
}

template <int NPL>
__device__ __forceinline__ void apply_gather(const int (&P)[NPL], const float (&D)[NPL],
                                             const float (&W)[NPL], float (&x)[NPL], float *sX,
                                             int N, int lane) {
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        if (e < N) sX[e] = x[r];
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < NPL; ++r) x[r] = W[r] + D[r] * sX[P[r]];
    __syncwarp();
}

// One CTA of nw warps per (b, h), or (G > 1) a cluster of G CTAs per
// sequence: the chunks are split over G * nw warps; each CTA reduces its
// warps' aggregates to a CTA total by a five-level tree, and warp 0 of CTA r
// starts from g_hlast advanced through the totals of CTAs G - 1 .. r + 1,
// read through distributed shared memory.
template <int NPL>
__global__ void k_bwdB(const ChunkParams p, int G) {
    extern __shared__ __align__(16) unsigned char sm_bb[];
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = (int)p.N;
    const int64_t bh = blockIdx.x / G;
    const int rank = G > 1 ? (int)cluster_rank() : 0;
    const int64_t C = p.C;
    float *sXall = reinterpret_cast<float *>(sm_bb);             // [nw][64]
    int *sPall = reinterpret_cast<int *>(sXall + nw * kMaxN);     // [nw][64]
    float *sDall = reinterpret_cast<float *>(sPall + nw * kMaxN); // [nw][64]
    int *aggP = reinterpret_cast<int *>(sDall + nw * kMaxN);
    float *aggD = reinterpret_cast<float *>(aggP + nw * kMaxN);
    float *aggW = aggD + nw * kMaxN;
    float *carry = aggW + nw * kMaxN;
    // G > 1: the reduction tree's aggregates [nw][64] (P, D, W); slot 0 ends
    // up with the CTA total
    int *treP = reinterpret_cast<int *>(carry + nw * kMaxN);
    float *treD = reinterpret_cast<float *>(treP + nw * kMaxN);
    float *treW = treD + nw * kMaxN;
    float *sX = sXall + warp * kMaxN;
    int *sP = sPall + warp * kMaxN;
    float *sD = sDall + warp * kMaxN;
    const int64_t gw = (int64_t)rank * nw + warp, nwt = (int64_t)G * nw;
    const int64_t c0 = C * gw / nwt, c1 = C * (gw + 1) / nwt;
    const int64_t u0 = bh * C;

    if (c0 < c1) {
        int aP[NPL];
        float aD[NPL], aW[NPL];
        load_rev<NPL>(p, u0 + c1 - 1, lane, aP, aD, aW);
        for (int64_t c = c1 - 2; c >= c0; --c) {
            int Pa[NPL];
            float Da[NPL], Wa[NPL];
            load_rev<NPL>(p, u0 + c, lane, Pa, Da, Wa);
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                if (e < N) {
                    sX[e] = aW[r];
                    sP[e] = aP[r];
                    sD[e] = aD[r];
                }
            }
            __syncwarp();
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int j = Pa[r];
                aW[r] = Wa[r] + Da[r] * sX[j];
                aD[r] = Da[r] * sD[j];
                aP[r] = sP[j];
            }
            __syncwarp();
        }
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            if (e < N) {
                aggP[warp * kMaxN + e] = aP[r];
                aggD[warp * kMaxN + e] = aD[r];
                aggW[warp * kMaxN + e] = aW[r];
            }
        }
    }
    __syncthreads();
    if (G > 1) {
        // the CTA total R_0 o R_1 o ... o R_{nw-1} (R_0 applied last): at
        // level d, warp w (w a multiple of 2d) composes its slot with slot
        // w + d: w = w_a + D_a * w_b[P_a], D = D_a * D_b[P_a], P = P_b[P_a].
        // Every warp's segment is non-empty (at least 64 chunks per CTA).
        int tP[NPL];
        float tD[NPL], tW[NPL];
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            tP[r] = e < N ? aggP[warp * kMaxN + e] : 0;
            tD[r] = e < N ? aggD[warp * kMaxN + e] : 0.f;
            tW[r] = e < N ? aggW[warp * kMaxN + e] : 0.f;
            if (e < N) {
                treP[warp * kMaxN + e] = tP[r];
                treD[warp * kMaxN + e] = tD[r];
                treW[warp * kMaxN + e] = tW[r];
            }
        }
        __syncthreads();
        for (int d = 1; d < nw; d <<= 1) {
            const bool active = (warp % (2 * d)) == 0 && warp + d < nw;
            if (active) {
                const int b0 = (warp + d) * kMaxN;
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    const int q = tP[r];
                    tW[r] = tW[r] + tD[r] * treW[b0 + q];
                    tD[r] = tD[r] * treD[b0 + q];
                    tP[r] = treP[b0 + q];
                }
            }
            __syncthreads();
            if (active) {
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    const int e = lane * NPL + r;
                    if (e < N) {
                        treP[warp * kMaxN + e] = tP[r];
                        treD[warp * kMaxN + e] = tD[r];
                        treW[warp * kMaxN + e] = tW[r];
                    }
                }
            }
            __syncthreads();
        }
        cluster_sync_all();   // every CTA's total (slot 0) is in place
    }
    if (warp == 0) {
        float x[NPL];
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            x[r] = (e < N && p.g_hlast) ? p.g_hlast[bh * p.N + e] : 0.f;
        }
        // the cluster's later CTAs, last first
        for (int q = G - 1; q > rank; --q) {
            int P[NPL];
            float D[NPL], W[NPL];
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                const int ee = e < N ? e : 0;
                P[r] = ldc_s32(cluster_map(smem_u32(treP + ee), (uint32_t)q));
                D[r] = ldc_f32(cluster_map(smem_u32(treD + ee), (uint32_t)q));
                W[r] = ldc_f32(cluster_map(smem_u32(treW + ee), (uint32_t)q));
                if (e >= N) {
                    P[r] = 0;
                    D[r] = 0.f;
                    W[r] = 0.f;
                }
            }
            apply_gather<NPL>(P, D, W, x, sX, N, lane);
        }
        for (int w = nw - 1; w >= 0; --w) {
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                if (e < N) carry[w * kMaxN + e] = x[r];
            }
            if (C * w / nw < C * (w + 1) / nw) {
                int P[NPL];
                float D[NPL], W[NPL];
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    const int e = lane * NPL + r;
                    P[r] = e < N ? aggP[w * kMaxN + e] : 0;
                    D[r] = e < N ? aggD[w * kMaxN + e] : 0.f;
                    W[r] = e < N ? aggW[w * kMaxN + e] : 0.f;
                }
                apply_gather<NPL>(P, D, W, x, sX, N, lane);
            }
        }
        if (p.g_h0 && rank == 0) {
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                const int e = lane * NPL + r;
                if (e < N) p.g_h0[bh * p.N + e] = x[r];
            }
        }
    }
    // every CTA is done reading the others' totals (G > 1); carries visible
    if (G > 1)
        cluster_sync_all();
    else
        __syncthreads();
    float x[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        x[r] = e < N ? carry[warp * kMaxN + e] : 0.f;
    }
    for (int64_t c = c1 - 1; c >= c0; --c) {
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            if (e < N) p.lam[(u0 + c) * p.N + e] = x[r];
        }
        int P[NPL];
        float D[NPL], W[NPL];
        load_rev<NPL>(p, u0 + c, lane, P, D, W);
        apply_gather<NPL>(P, D, W, x, sX, N, lane);
    }
}

// ---------------------------------------------------------------------------
// bwd phase C: per chunk, (1) forward recompute from H_{c-1} keeping the
// state at every tile start in shared memory, (2) per tile in reverse:
// recompute the tile's states into shared memory, then sweep back emitting
// g_b = lambda, g_c = g_y h, g_d = h_{t-1} * lambda[pi(.)].
// ---------------------------------------------------------------------------
template <typename T, int NPL, bool FULL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_bwdC(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_bc[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_bc, warp, lane);
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int N = (int)p.N, K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    unsigned char *wbase = sm_bc + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    const int rowb = N * (int)sizeof(T);
    Ring<3> ring;
    ring.buf = wbase;
    ring.rowb = rowb;
    ring.esz = (int)sizeof(T);
    ring.tens_bytes = kTS * rowb;
    ring.stage_bytes = 3 * ring.tens_bytes;
    ring.ns = p.ns;
    ring.bulk = p.bulk != 0;
    float *pbuf = reinterpret_cast<float *>(wbase + p.ns * ring.stage_bytes);
    float *lbuf = pbuf + 2 * kPbStride + kYbufFloats;
    float *ck = lbuf + 2 * kPbStride;                 // [kBwdMaxChunk / kTS][64]
    float *hsm = ck + (kBwdMaxChunk / kTS) * kMaxN;   // [kTS + 1][64]
    ring.bar0 = smem_u32(hsm + (kTS + 1) * kMaxN);
    const int64_t seq_row0 = bh * p.L;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + seq_row0 * rowb;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.b) + seq_row0 * rowb;
    ring.src[2] = reinterpret_cast<const unsigned char *>(p.c) + seq_row0 * rowb;
    ring_init_bars(ring.bar0, p.ns, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    const int total = 2 * ntiles;   // pass 1 tiles, then pass 2 tiles (reverse)
    auto tile_of = [&](int m) { return m < ntiles ? m : 2 * ntiles - 1 - m; };
    auto nt_of = [&](int m) { return m < ntiles ? 2 : 3; };
    for (int m = 0; m < p.ns && m < total; ++m) {
        const int ti = tile_of(m);
        ring.issue(m, s + (int64_t)ti * kTS, min(kTS, len - ti * kTS), nt_of(m), lane);
    }
    for (int m = p.ns; m < p.ns + kPrefetchTiles && m < ntiles; ++m)
        ring.prefetch(s + (int64_t)m * kTS, min(kTS, len - m * kTS), 3, lane);
    clear_pb(pbuf, lane);

    const int32_t *kp = p.k + bh * p.L + s;
    const float *gyp = p.g_y + bh * p.L + s;
    float h[NPL], mu[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        h[r] = 0.f;
        mu[r] = 0.f;
        if (e < N) {
            h[r] = cidx == 0 ? (p.h0 ? p.h0[bh * p.N + e] : 0.f) : p.Hc[(unit - 1) * p.N + e];
            mu[r] = p.lam[unit * p.N + e];
        }
    }
    int kreg = load_k(kp, lane, lane < kTS && lane < len, K, p.status);
    float gyreg = 0.f;

    for (int m = 0; m < total; ++m) {
        const int stage = m % p.ns;
        if (!ring.wait(stage, (uint32_t)((m / p.ns) & 1))) {
            ring_abort(ring, m, min(total, m + p.ns), p.status, lane);
            return;
        }
        const int ti = tile_of(m);
        const int t0 = ti * kTS;
        const int n = min(kTS, len - t0);
        int knext = 0;
        float gynext = 0.f;
        if (m + 1 < total) {
            const int tn0 = tile_of(m + 1) * kTS;
            const bool v = lane < kTS && tn0 + lane < len;
            knext = load_k_raw(kp, tn0 + lane, v);
            if (m + 1 >= ntiles) gynext = v ? gyp[tn0 + lane] : 0.f;
        }
        const T *td = reinterpret_cast<const T *>(ring.tile(stage, 0));
        const T *tb = reinterpret_cast<const T *>(ring.tile(stage, 1));
        const T *tc = reinterpret_cast<const T *>(ring.tile(stage, 2));
        if (m < ntiles) {
            // pass 1: checkpoint at the tile start, then advance the state
            st_own<NPL, FULL>(ck + ti * kMaxN, lane, N, h);
#pragma unroll 2
            for (int q = 0; q < n; ++q) {
                const int kk = __shfl_sync(kFull, kreg, q);
                float dv[NPL], bv[NPL];
                ld_own<T, NPL, FULL>(td + q * N, lane, N, dv);
                ld_own<T, NPL, FULL>(tb + q * N, lane, N, bv);
                pd_gather_step<NPL, FULL>(h, dv, bv, pbuf + (q & 1) * kPbStride,
                                          sd.tab + kk * (kDcap * 64) + lane * NPL, sd.fan[kk],
                                          sd.map + kk * N, lane, N);
            }
        } else {
            // pass 2: states of this tile, hsm[q] = h_{t0+q-1}
            float x[NPL];
            ld_own<float, NPL, FULL>(ck + ti * kMaxN, lane, N, x);
            st_own<NPL, FULL>(hsm, lane, N, x);
#pragma unroll 2
            for (int q = 0; q < n; ++q) {
                const int kk = __shfl_sync(kFull, kreg, q);
                float dv[NPL], bv[NPL];
                ld_own<T, NPL, FULL>(td + q * N, lane, N, dv);
                ld_own<T, NPL, FULL>(tb + q * N, lane, N, bv);
                pd_gather_step<NPL, FULL>(x, dv, bv, pbuf + (q & 1) * kPbStride,
                                          sd.tab + kk * (kDcap * 64) + lane * NPL, sd.fan[kk],
                                          sd.map + kk * N, lane, N);
                st_own<NPL, FULL>(hsm + (q + 1) * kMaxN, lane, N, x);
            }
#pragma unroll 2
            for (int q = n - 1; q >= 0; --q) {
                const int kk = __shfl_sync(kFull, kreg, q);
                const float gy = __shfl_sync(kFull, gyreg, q);
                const int64_t row = (int64_t)(t0 + q) * p.N;
                float dv[NPL], cv[NPL], hq[NPL], hp[NPL], lam[NPL], gc[NPL], gd[NPL];
                ld_own<T, NPL, FULL>(td + q * N, lane, N, dv);
                ld_own<T, NPL, FULL>(tc + q * N, lane, N, cv);
                ld_own<float, NPL, FULL>(hsm + (q + 1) * kMaxN, lane, N, hq);
                ld_own<float, NPL, FULL>(hsm + q * kMaxN, lane, N, hp);
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    lam[r] = gy * cv[r] + mu[r];
                    gc[r] = gy * hq[r];
                }
                float *lb = lbuf + (q & 1) * kPbStride;
                st_own<NPL, FULL>(lb, lane, N, lam);
                st_own<NPL, FULL>(p.g_b + seq_row0 * p.N + s * p.N + row, lane, N, lam);
                st_own<NPL, FULL>(p.g_c + seq_row0 * p.N + s * p.N + row, lane, N, gc);
                __syncwarp();
                int tgt[NPL];
                own_targets2<NPL, FULL>(sd.map + kk * N, lane, N, tgt);
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    const float gl = lb[tgt[r]];
                    gd[r] = hp[r] * gl;
                    mu[r] = dv[r] * gl;
                }
                st_own<NPL, FULL>(p.g_d + seq_row0 * p.N + s * p.N + row, lane, N, gd);
            }
        }
        __syncwarp();
        if (m + p.ns < total) {
            const int mn = m + p.ns;
            const int tn = tile_of(mn);
            ring.issue(stage, s + (int64_t)tn * kTS, min(kTS, len - tn * kTS), nt_of(mn), lane);
        }
        if (m + p.ns + kPrefetchTiles < ntiles) {
            const int tp2 = m + p.ns + kPrefetchTiles;
            ring.prefetch(s + (int64_t)tp2 * kTS, min(kTS, len - tp2 * kTS), 3, lane);
        }
        kreg = clamp_k(knext, K, p.status);
        gyreg = gynext;
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <typename KernT>
static cudaError_t launch_chunk_b(KernT kern, const ChunkParams &p, size_t, cudaStream_t st) {
    return launch_units(kern, p, p.smem_per_warp, st);
}

#define PDSSM_DISPATCH_B(KERNEL, p, st, smem)                                     \
    do {                                                                         \
        if ((p).N == 64) return launch_chunk_b(KERNEL<T, 2, true>, p, smem, st); \
        if ((p).N > 32) return launch_chunk_b(KERNEL<T, 2, false>, p, smem, st); \
        if ((p).N == 32) return launch_chunk_b(KERNEL<T, 1, true>, p, smem, st); \
        return launch_chunk_b(KERNEL<T, 1, false>, p, smem, st);                 \
    } while (0)

template <typename T>
static cudaError_t bwdA_t(ChunkParams p, cudaStream_t st) {
    const int rowb = (int)p.N * (int)sizeof(T);
    p.smem_per_warp = warp_smem_bytes(p.ns, 2, rowb);
    const size_t smem = 0;
    PDSSM_DISPATCH_B(k_bwdA, p, st, smem);
}

template <typename T>
static cudaError_t bwdC_t(ChunkParams p, cudaStream_t st) {
    const int rowb = (int)p.N * (int)sizeof(T);
    p.smem_per_warp = bwd_warp_smem_bytes(p.ns, 3, rowb);
    const size_t smem = 0;
    PDSSM_DISPATCH_B(k_bwdC, p, st, smem);
}

cudaError_t launch_bwdA(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st) {
    if (p.units == 0) return cudaSuccess;
    if (fast_path(p)) return launch_bwdA_fast(p, dt, st);
    return dt == PDSSM_BF16 ? bwdA_t<__nv_bfloat16>(p, st) : bwdA_t<float>(p, st);
}

cudaError_t launch_bwdC(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st) {
    if (p.units == 0) return cudaSuccess;
    if (fast_path(p)) return launch_bwdC_fast(p, dt, st);
    return dt == PDSSM_BF16 ? bwdC_t<__nv_bfloat16>(p, st) : bwdC_t<float>(p, st);
}

template <int NPL>
static cudaError_t launch_bwdB_t(const ChunkParams &p, int nw, int G, cudaStream_t st) {
    const size_t smem = (size_t)nw * kMaxN * 4 * (G > 1 ? 10 : 7);
    const int64_t BH = p.B * p.H;
    cudaError_t e =
        cudaFuncSetAttribute(k_bwdB<NPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (G > 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(BH * G));
        cfg.blockDim = dim3(nw * 32);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)G;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, k_bwdB<NPL>, p, G);
    }
    k_bwdB<NPL><<<(unsigned)BH, nw * 32, smem, st>>>(p, G);
    return cudaGetLastError();
}

cudaError_t launch_bwdB(const ChunkParams &p, cudaStream_t st) {
    if (p.units == 0) return cudaSuccess;
    const int nw = (int)imin64(32, p.C);
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int G = carry_scan_cluster(p.B * p.H, p.C, sms);
    return p.N > 32 ? launch_bwdB_t<2>(p, nw, G, st) : launch_bwdB_t<1>(p, nw, G, st);
}

}  // namespace pdssm
