// Backward phases A and C for a state that fills the warp (N = 32 or 64),
// the arithmetic of bwd.cu written against explicit 32-bit shared addresses
// (dictionary staged as byte offsets; targets fetched before the warp
// barrier; the forward recompute uses the fan-in-class slot gather).
#include "common.cuh"

namespace pdssm {

template <int NPL>
__device__ __forceinline__ void sts_own(uint32_t a, const float (&v)[NPL]) {
    if constexpr (NPL == 1)
        sts_f32(a, v[0]);
    else
        sts_f32x2(a, v[0], v[1]);
}

template <int NPL>
__device__ __forceinline__ void targets4(uint32_t a, int (&t4)[NPL]) {
    if constexpr (NPL == 1) {
        t4[0] = lds_s32(a);
    } else {
        const int2 q = lds_s32x2(a);
        t4[0] = q.x;
        t4[1] = q.y;
    }
}

template <int NPL>
__device__ __forceinline__ void stg_own(float *row, int lane, const float (&v)[NPL]) {
    if constexpr (NPL == 1)
        row[lane] = v[0];
    else
        *reinterpret_cast<float2 *>(row + 2 * lane) = make_float2(v[0], v[1]);
}

// ---------------------------------------------------------------------------
// bwd phase A: w_c = M_s^T lambda^loc_s from a zero carry
// ---------------------------------------------------------------------------
template <typename T, int NPL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_bwdA_fast(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_ba[];
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int TENS = kTS * ROWB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_ba, warp, lane, 4);
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    unsigned char *wbase = sm_ba + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    Ring<2> ring;
    ring.buf = wbase;
    ring.rowb = ROWB;
    ring.esz = (int)sizeof(T);
    ring.tens_bytes = TENS;
    ring.stage_bytes = 2 * TENS;
    ring.ns = p.ns;
    ring.bulk = p.bulk != 0;
    float *lbuf = reinterpret_cast<float *>(wbase + p.ns * ring.stage_bytes);
    ring.bar0 = smem_u32(lbuf + 2 * kPbStride + kYbufFloats);
    const int64_t seq_row0 = bh * p.L;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + seq_row0 * ROWB;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.c) + seq_row0 * ROWB;
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
    const uint32_t map_s = smem_u32(sd.map), lb_s = smem_u32(lbuf);
    const uint32_t own_off = lane * NPL * (uint32_t)sizeof(T);
    const int32_t *kp = p.k + seq_row0 + s;
    const float *gyp = p.g_y + seq_row0 + s;
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
        uint32_t row = smem_u32(ring.tile(stage, 0)) + (n - 1) * ROWB;
        for (int q = n - 1; q >= 0; --q, row -= ROWB) {
            const int kk = __shfl_sync(kFull, kreg, q);
            const float gy = __shfl_sync(kFull, gyreg, q);
            float dv[NPL], cv[NPL], lam[NPL];
            int t4[NPL];
            lds_own<T, NPL>(row + own_off, dv);
            lds_own<T, NPL>(row + own_off + TENS, cv);
            targets4<NPL>(map_s + kk * (N * 4) + lane * NPL * 4, t4);
#pragma unroll
            for (int r = 0; r < NPL; ++r) lam[r] = gy * cv[r] + mu[r];
            const uint32_t lb = lb_s + (q & 1) * (kPbStride * 4);
            sts_own<NPL>(lb + lane * NPL * 4, lam);
            warp_barrier();
#pragma unroll
            for (int r = 0; r < NPL; ++r) mu[r] = dv[r] * lds_f32(lb + t4[r]);
        }
        warp_barrier();
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
    for (int r = 0; r < NPL; ++r) p.wc[o + lane * NPL + r] = mu[r];
}

// ---------------------------------------------------------------------------
// bwd phase C: forward recompute with checkpoints, then per tile in reverse:
// recompute the tile's states, sweep back emitting g_b, g_c, g_d.
// ---------------------------------------------------------------------------
constexpr int kBwdFastExtraFloats =
    2 * kPbStride + (kBwdMaxChunk / kTS) * kMaxN + (kTS + 1) * kMaxN;

template <typename T, int NPL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_bwdC_fast(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_bc[];
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int TENS = kTS * ROWB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_bc, warp, lane, 4);
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    unsigned char *wbase = sm_bc + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    Ring<3> ring;
    ring.buf = wbase;
    ring.rowb = ROWB;
    ring.esz = (int)sizeof(T);
    ring.tens_bytes = TENS;
    ring.stage_bytes = 3 * TENS;
    ring.ns = p.ns;
    ring.bulk = p.bulk != 0;
    float *pbuf = reinterpret_cast<float *>(wbase + p.ns * ring.stage_bytes);
    float *lbuf = pbuf + 2 * kPbStride + kYbufFloats;
    float *ck = lbuf + 2 * kPbStride;                 // [kBwdMaxChunk / kTS][64]
    float *hsm = ck + (kBwdMaxChunk / kTS) * kMaxN;   // [kTS + 1][64]
    ring.bar0 = smem_u32(hsm + (kTS + 1) * kMaxN);
    const int64_t seq_row0 = bh * p.L;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + seq_row0 * ROWB;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.b) + seq_row0 * ROWB;
    ring.src[2] = reinterpret_cast<const unsigned char *>(p.c) + seq_row0 * ROWB;
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

    const uint32_t map_s = smem_u32(sd.map), fan_s = smem_u32(sd.fan);
    const uint32_t tab_lane = smem_u32(sd.tab) + lane * NPL;
    const uint32_t pb_s = smem_u32(pbuf), lb_s = smem_u32(lbuf);
    const uint32_t ck_lane = smem_u32(ck) + lane * NPL * 4;
    const uint32_t hs_lane = smem_u32(hsm) + lane * NPL * 4;
    const uint32_t own_off = lane * NPL * (uint32_t)sizeof(T);
    const int32_t *kp = p.k + seq_row0 + s;
    const float *gyp = p.g_y + seq_row0 + s;
    float *gb = p.g_b + (seq_row0 + s) * N;
    float *gc = p.g_c + (seq_row0 + s) * N;
    float *gd = p.g_d + (seq_row0 + s) * N;

    float h[NPL], mu[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        h[r] = cidx == 0 ? (p.h0 ? p.h0[bh * N + e] : 0.f) : p.Hc[(unit - 1) * N + e];
        mu[r] = p.lam[unit * N + e];
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
        const uint32_t tile = smem_u32(ring.tile(stage, 0));
        if (m < ntiles) {
            // pass 1: checkpoint at the tile start, then advance the state
            sts_own<NPL>(ck_lane + ti * (kMaxN * 4), h);
            uint32_t row = tile;
            for (int q = 0; q < n; ++q, row += ROWB) {
                const int kk = __shfl_sync(kFull, kreg, q);
                float dv[NPL], bv[NPL];
                lds_own<T, NPL>(row + own_off, dv);
                lds_own<T, NPL>(row + own_off + TENS, bv);
                step_any<NPL>(h, dv, bv, pb_s + (q & 1) * (kPbStride * 4),
                              tab_lane + kk * (kDcap * 64), lds_s32(fan_s + kk * 4),
                              map_s + kk * (N * 4), lane);
            }
        } else {
            // pass 2: states of this tile, hsm[q] = h_{t0+q-1}
            float x[NPL];
            lds_own<float, NPL>(ck_lane + ti * (kMaxN * 4), x);
            sts_own<NPL>(hs_lane, x);
            uint32_t row = tile;
            for (int q = 0; q < n; ++q, row += ROWB) {
                const int kk = __shfl_sync(kFull, kreg, q);
                float dv[NPL], bv[NPL];
                lds_own<T, NPL>(row + own_off, dv);
                lds_own<T, NPL>(row + own_off + TENS, bv);
                step_any<NPL>(x, dv, bv, pb_s + (q & 1) * (kPbStride * 4),
                              tab_lane + kk * (kDcap * 64), lds_s32(fan_s + kk * 4),
                              map_s + kk * (N * 4), lane);
                sts_own<NPL>(hs_lane + (q + 1) * (kMaxN * 4), x);
            }
            row = tile + (n - 1) * ROWB;
            for (int q = n - 1; q >= 0; --q, row -= ROWB) {
                const int kk = __shfl_sync(kFull, kreg, q);
                const float gy = __shfl_sync(kFull, gyreg, q);
                float dv[NPL], cv[NPL], hq[NPL], hp[NPL], lam[NPL], gcv[NPL], gdv[NPL];
                int t4[NPL];
                lds_own<T, NPL>(row + own_off, dv);
                lds_own<T, NPL>(row + own_off + 2 * TENS, cv);
                lds_own<float, NPL>(hs_lane + (q + 1) * (kMaxN * 4), hq);
                lds_own<float, NPL>(hs_lane + q * (kMaxN * 4), hp);
                targets4<NPL>(map_s + kk * (N * 4) + lane * NPL * 4, t4);
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    lam[r] = gy * cv[r] + mu[r];
                    gcv[r] = gy * hq[r];
                }
                const uint32_t lb = lb_s + (q & 1) * (kPbStride * 4);
                sts_own<NPL>(lb + lane * NPL * 4, lam);
                const int64_t ro = (int64_t)(t0 + q) * N;
                stg_own<NPL>(gb + ro, lane, lam);
                stg_own<NPL>(gc + ro, lane, gcv);
                warp_barrier();
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    const float gl = lds_f32(lb + t4[r]);
                    gdv[r] = hp[r] * gl;
                    mu[r] = dv[r] * gl;
                }
                stg_own<NPL>(gd + ro, lane, gdv);
            }
        }
        warp_barrier();
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

template <typename KernT>
static cudaError_t launch_bfast(KernT kern, const ChunkParams &p, size_t, cudaStream_t st) {
    return launch_units(kern, p, p.smem_per_warp, st);
}

cudaError_t launch_bwdA_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.smem_per_warp = warp_smem_bytes(p.ns, 2, (int)p.N * es);
    const size_t smem = 0;
    if (dt == PDSSM_BF16)
        return p.N == 64 ? launch_bfast(k_bwdA_fast<__nv_bfloat16, 2>, p, smem, st)
                         : launch_bfast(k_bwdA_fast<__nv_bfloat16, 1>, p, smem, st);
    return p.N == 64 ? launch_bfast(k_bwdA_fast<float, 2>, p, smem, st)
                     : launch_bfast(k_bwdA_fast<float, 1>, p, smem, st);
}

cudaError_t launch_bwdC_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.smem_per_warp = warp_smem_bytes(p.ns, 3, (int)p.N * es, kBwdFastExtraFloats * 4);
    const size_t smem = 0;
    if (dt == PDSSM_BF16)
        return p.N == 64 ? launch_bfast(k_bwdC_fast<__nv_bfloat16, 2>, p, smem, st)
                         : launch_bfast(k_bwdC_fast<__nv_bfloat16, 1>, p, smem, st);
    return p.N == 64 ? launch_bfast(k_bwdC_fast<float, 2>, p, smem, st)
                     : launch_bfast(k_bwdC_fast<float, 1>, p, smem, st);
}

}  // namespace pdssm
