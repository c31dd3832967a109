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
#include "transfer_ops.cuh"

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
// phase B: G CTAs of nw warps per (b, h) (G > 1: one thread-block cluster
// per sequence).  Chunks are split into G * nw contiguous segments: (1) each
// warp composes its segment's transfers into one aggregate, (2) the
// aggregates of a CTA are combined by an inclusive Hillis-Steele scan
// (log2 nw rounds); with G > 1 each CTA publishes its total in shared memory
// and, after a cluster barrier, warp 0 of CTA r applies the totals of CTAs
// 0 .. r - 1, read through distributed shared memory, to h0, which gives the
// CTA's carry-in; the scan applied to the carry-in gives every segment's
// carry, (3) each warp re-applies its segment's transfers from its carry
// and stores every H_c.  Transfers are held in the layout of
// transfer_ops.cuh (lane l: elements l and l + 32).
// ---------------------------------------------------------------------------

constexpr int kBGroup = 2;   // transfers loaded together

__global__ void __launch_bounds__(1024, 1) k_phaseB(const ChunkParams p, int G) {
    extern __shared__ __align__(16) unsigned char sm_b[];
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();   // the chunk transfers come from the preceding kernel
    const int64_t bh = blockIdx.x / G;
    const int rank = G > 1 ? (int)cluster_rank() : 0;
    const int64_t C = p.C;
    const bool perm = __ldg(p.dict_stats + 1) <= 1;   // every map a permutation
    // [2 buffers][nw][64] aggregates, [nw][64] carries, [nw] scratch, this
    // CTA's total (P, D, V) and its carry-in
    int *aggP = reinterpret_cast<int *>(sm_b);
    float *aggD = reinterpret_cast<float *>(aggP + 2 * nw * 64);
    float *aggV = aggD + 2 * nw * 64;
    float *carry = aggV + 2 * nw * 64;
    ScatterScratch *scr = reinterpret_cast<ScatterScratch *>(carry + nw * 64);
    ScatterScratch &sc = scr[warp];
    int *totP = reinterpret_cast<int *>(scr + nw);
    float *totD = reinterpret_cast<float *>(totP + 64);
    float *totV = totD + 64;
    float *xin = totV + 64;
    // the staged chunk transfer of the level-1 gathers reuses key / val
    int *tP = sc.key;
    float *tD = sc.val;

    const int64_t gw = (int64_t)rank * nw + warp, nwt = (int64_t)G * nw;
    const int64_t c0 = C * gw / nwt, c1 = C * (gw + 1) / nwt;
    const int64_t u0 = bh * C;

    // (1) segment aggregate T_{c1-1} o ... o T_{c0}; identity for an empty segment
    Agg a;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        a.P[r] = e < p.N ? e : kPadIdx;
        a.D[r] = e < p.N ? 1.f : 0.f;
        a.V[r] = 0.f;
    }
    for (int64_t g = c0; g < c1; g += kBGroup) {
        int TP[kBGroup][2];
        float TD[kBGroup][2], TV[kBGroup][2];
#pragma unroll
        for (int i = 0; i < kBGroup; ++i)
            if (g + i < c1) load_transfer2(p, u0 + g + i, lane, TP[i], TD[i], TV[i]);
#pragma unroll
        for (int i = 0; i < kBGroup; ++i) {
            if (g + i >= c1) break;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                tP[lane + 32 * r] = TP[i][r];
                tD[lane + 32 * r] = TD[i][r];
            }
            __syncwarp();
            // the gathers read tP / tD before the scatter overwrites them
            int gP[2];
            float gD[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                gP[r] = tP[a.P[r]];
                gD[r] = tD[a.P[r]];
            }
            __syncwarp();
            float z[2], nv[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) z[r] = TD[i][r] * a.V[r];
            warp_scatter(TP[i], z, TV[i], nv, sc, lane, perm);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                a.D[r] *= gD[r];
                a.P[r] = gP[r];
                a.V[r] = nv[r];
            }
        }
    }
    // (2) inclusive scan of the aggregates: after round d, warp w holds
    // A_w o A_{w-1} o ... o A_{max(0, w - 2d + 1)}
    int cur = 0;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        aggP[(cur * nw + warp) * 64 + e] = a.P[r];
        aggD[(cur * nw + warp) * 64 + e] = a.D[r];
        aggV[(cur * nw + warp) * 64 + e] = a.V[r];
    }
    __syncthreads();
    for (int d = 1; d < nw; d <<= 1) {
        if (warp >= d) {
            // this warp's aggregate goes after warp (warp - d)'s
            const int src = (cur * nw + warp - d) * 64;
            Agg lo;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int e = lane + 32 * r;
                lo.P[r] = aggP[src + e];
                lo.D[r] = aggD[src + e];
                lo.V[r] = aggV[src + e];
            }
            const int *hP = aggP + (cur * nw + warp) * 64;
            const float *hD = aggD + (cur * nw + warp) * 64;
            compose_after(lo, hP, hD, a.P, a.D, a.V, sc, lane, perm);
            a = lo;
        }
        const int nxt = cur ^ 1;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            aggP[(nxt * nw + warp) * 64 + e] = a.P[r];
            aggD[(nxt * nw + warp) * 64 + e] = a.D[r];
            aggV[(nxt * nw + warp) * 64 + e] = a.V[r];
        }
        cur = nxt;
        __syncthreads();
    }
    // the CTA's carry-in: h0, advanced (G > 1) through the totals of the
    // cluster's earlier CTAs
    if (G > 1) {
        if (warp == nw - 1) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int e = lane + 32 * r;
                totP[e] = a.P[r];
                totD[e] = a.D[r];
                totV[e] = a.V[r];
            }
        }
        cluster_sync_all();
        if (warp == 0) {
            float x[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int e = lane + 32 * r;
                x[r] = p.h0 && e < p.N ? p.h0[bh * p.N + e] : 0.f;
            }
            for (int q = 0; q < rank; ++q) {
                int P[2];
                float D[2], V[2], z[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int e = lane + 32 * r;
                    P[r] = ldc_s32(cluster_map(smem_u32(totP + e), (uint32_t)q));
                    D[r] = ldc_f32(cluster_map(smem_u32(totD + e), (uint32_t)q));
                    V[r] = ldc_f32(cluster_map(smem_u32(totV + e), (uint32_t)q));
                    z[r] = D[r] * x[r];
                }
                warp_scatter(P, z, V, x, sc, lane, perm);
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) xin[lane + 32 * r] = x[r];
        }
        // every CTA is done reading the others' totals, and xin is visible
        cluster_sync_all();
    }
    // carry at the end of this warp's segment: (prefix aggregate)(carry-in)
    float S[2];
    if (G > 1 || p.h0) {
        float z[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            z[r] = a.D[r] * (G > 1 ? xin[e] : (e < p.N ? p.h0[bh * p.N + e] : 0.f));
        }
        warp_scatter(a.P, z, a.V, S, sc, lane, perm);
    } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) S[r] = a.V[r];
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) carry[warp * 64 + lane + 32 * r] = S[r];
    if (warp == nw - 1 && rank == G - 1 && p.h_last) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            if (e < p.N) p.h_last[bh * p.N + e] = S[r];
        }
    }
    __syncthreads();
    // (3) re-apply this warp's transfers from its carry-in, storing every H_c
    float x[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        x[r] = warp > 0 ? carry[(warp - 1) * 64 + e]
                        : (G > 1 ? xin[e] : (p.h0 && e < p.N ? p.h0[bh * p.N + e] : 0.f));
    }
    for (int64_t g = c0; g < c1; g += kBGroup) {
        int TP[kBGroup][2];
        float TD[kBGroup][2], TV[kBGroup][2];
#pragma unroll
        for (int i = 0; i < kBGroup; ++i)
            if (g + i < c1) load_transfer2(p, u0 + g + i, lane, TP[i], TD[i], TV[i]);
#pragma unroll
        for (int i = 0; i < kBGroup; ++i) {
            if (g + i >= c1) break;
            float z[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) z[r] = TD[i][r] * x[r];
            warp_scatter(TP[i], z, TV[i], x, sc, lane, perm);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int e = lane + 32 * r;
                if (e < p.N) p.Hc[(u0 + g + i) * p.N + e] = x[r];
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
    const size_t smem =
        (size_t)nw * 64 * 4 * 7 + (size_t)nw * sizeof(ScatterScratch) + (size_t)4 * 64 * 4;
    const int64_t BH = p.B * p.H;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int G = carry_scan_cluster(BH, p.C, sms);
    e = cudaFuncSetAttribute(k_phaseB, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (G > 1)
        return launch_cluster_pdl(k_phaseB, dim3((unsigned)(BH * G)), dim3(nw * 32), smem, G, st,
                                  p, G);
    return launch_pdl(k_phaseB, dim3((unsigned)BH), dim3(nw * 32), smem, st, p, G);
}

}  // namespace pdssm
