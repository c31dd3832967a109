// Backward phases A and C for a state that fills the warp (N = 32 or 64),
// the arithmetic of bwd.cu written against explicit 32-bit shared addresses
// (dictionary staged as byte offsets; targets fetched before the warp
// barrier; the forward recompute uses the segment-table step).
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

// this lane's entries of a row written earlier by this same lane (plain
// loads: the data was written inside this kernel)
template <int NPL>
__device__ __forceinline__ void ldg_own(const float *row, int lane, float (&v)[NPL]) {
    if constexpr (NPL == 1) {
        v[0] = row[lane];
    } else {
        const float2 q = *reinterpret_cast<const float2 *>(row + 2 * lane);
        v[0] = q.x;
        v[1] = q.y;
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
    extern __shared__ __align__(128) unsigned char sm_ba_raw[];
    unsigned char *sm_ba = smem_base256(sm_ba_raw);
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
    using RingT = FastRing<2, ROWB>;
    float *lbuf = reinterpret_cast<float *>(wbase + kFastStages * RingT::STAGEB);
    RingT ring;
    ring.ring_s = smem_u32(wbase);
    ring.bar0 = smem_u32(lbuf + 2 * kPbStride);
    ring.len = len;
    ring.nt = 2;
    const int64_t row0 = bh * p.L + s;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + row0 * ROWB;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.c) + row0 * ROWB;
    ring_init_bars(ring.bar0, kFastStages, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    // tiles in reverse order: slot j holds chunk tile ntiles - 1 - j
    for (int j = 0; j < kFastStages && j < ntiles; ++j) ring.issue_tile(j, ntiles - 1 - j, 3u, lane);
    const uint32_t map_s = smem_u32(sd.map), lb_s = smem_u32(lbuf);
    const uint32_t own_off = lane * NPL * (uint32_t)sizeof(T);
    const int32_t *kp = p.k + row0;
    const float *gyp = p.g_y + row0;
    float mu[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) mu[r] = 0.f;
    int t0 = (ntiles - 1) * kTS;
    int kreg = load_k(kp, t0 + lane, lane < kTS && t0 + lane < len, K, p.status);
    float gyreg = (lane < kTS && t0 + lane < len) ? gyp[t0 + lane] : 0.f;

    for (int j = 0; j < ntiles; ++j) {
        if (!ring.wait(j)) {
            ring.abort(j, ntiles, p.status, lane);
            return;
        }
        t0 = (ntiles - 1 - j) * kTS;
        const int n = min(kTS, len - t0);
        const int tp = t0 - kTS;   // the tile processed next
        const bool vp = lane < kTS && tp >= 0;
        const int knext = load_k_raw(kp, tp + lane, vp);
        const float gynext = vp ? gyp[tp + lane] : 0.f;
        uint32_t row = ring.tile(j) + (n - 1) * ROWB;
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
        if (j + kFastStages < ntiles) ring.issue_tile(j + kFastStages, ntiles - 1 - (j + kFastStages), 3u, lane);
        kreg = clamp_k(knext, K, p.status);
        gyreg = gynext;
    }
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < NPL; ++r) p.wc[o + lane * NPL + r] = mu[r];
}

// ---------------------------------------------------------------------------
// bwd phase C: pass 1 runs the chunk forward from its carry and leaves every
// state h_t in g_c's row t; pass 2 takes the tiles in reverse, reads each
// tile's states back (prefetched one tile ahead) and sweeps back emitting
// g_b, g_c, g_d.  Step t of the sweep reads rows t and t - 1 of g_c and then
// overwrites row t with its gradient; rows below t are still states.
// ---------------------------------------------------------------------------
constexpr int kBwdFastExtraFloats = 2 * kPbStride + (kTS + 1) * kMaxN;

template <typename T, int NPL, int LV>
__device__ __forceinline__ void bwdC_fast_unit(const ChunkParams &p, const SmemDict &sd,
                                               unsigned char *wbase, int64_t unit, int lane) {
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int TENS = kTS * ROWB;
    const int K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    // two tensors per stage: d, then b (pass 1) or c (pass 2) in the second
    // slot, so a warp's ring is 2/3 of three slots and more warps fit an SM
    using RingT = FastRing<2, ROWB>;
    float *pbuf = reinterpret_cast<float *>(wbase + kFastStages * RingT::STAGEB);
    float *lbuf = pbuf + 2 * kPbStride;
    float *hsm = lbuf + 2 * kPbStride;                // [kTS + 1][64]
    RingT ring;
    ring.ring_s = smem_u32(wbase);
    ring.bar0 = smem_u32(hsm + (kTS + 1) * kMaxN);
    ring.len = len;
    ring.nt = 2;
    const int64_t row0 = bh * p.L + s;
    const unsigned char *src_b = reinterpret_cast<const unsigned char *>(p.b) + row0 * ROWB;
    const unsigned char *src_c = reinterpret_cast<const unsigned char *>(p.c) + row0 * ROWB;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + row0 * ROWB;
    ring.src[1] = src_b;
    ring_init_bars(ring.bar0, kFastStages, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    const int total = 2 * ntiles;   // pass 1 tiles, then pass 2 tiles (reverse)
    auto tile_of = [&](int m) { return m < ntiles ? m : 2 * ntiles - 1 - m; };
    // pass 1 stages d and b, pass 2 d and c
    auto issue = [&](int m) {
        ring.src[1] = m < ntiles ? src_b : src_c;
        ring.issue_tile(m, tile_of(m), 3u, lane);
    };
    for (int m = 0; m < kFastStages && m < total; ++m) issue(m);

    const uint32_t map_s = smem_u32(sd.map);
    const uint32_t seg_lane = smem_u32(sd.seg) + lane * 8;
    const uint32_t pb_s = smem_u32(pbuf), ob_s = pb_s + 256, lb_s = smem_u32(lbuf);   // pb, ob 256-byte aligned
    const uint32_t hs_lane = smem_u32(hsm) + lane * NPL * 4;
    const uint32_t own_off = lane * NPL * (uint32_t)sizeof(T);
    const int32_t *kp = p.k + row0;
    const float *gyp = p.g_y + row0;
    float *gb = p.g_b + row0 * N;
    float *gc = p.g_c + row0 * N;
    float *gd = p.g_d + row0 * N;

    float h[NPL], hinit[NPL], mu[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        h[r] = cidx == 0 ? (p.h0 ? p.h0[bh * N + e] : 0.f) : p.Hc[(unit - 1) * N + e];
        hinit[r] = h[r];
        mu[r] = p.lam[unit * N + e];
    }
    // states of the next pass-2 tile, rows t0 - 1 .. t0 + n - 1
    float nst[kTS + 1][NPL];
    auto load_states = [&](int ti2) {
        const int t02 = ti2 * kTS, n2 = min(kTS, len - t02);
#pragma unroll
        for (int q = 0; q <= kTS; ++q) {
            if (q > n2) break;
            if (q == 0 && t02 == 0) {
#pragma unroll
                for (int r = 0; r < NPL; ++r) nst[0][r] = hinit[r];
            } else {
                ldg_own<NPL>(gc + (int64_t)(t02 + q - 1) * N, lane, nst[q]);
            }
        }
    };
    int kreg = load_k(kp, lane, lane < kTS && lane < len, K, p.status);
    float gyreg = 0.f;

    for (int m = 0; m < total; ++m) {
        if (!ring.wait(m)) {
            ring.abort(m, total, p.status, lane);
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
        const uint32_t tile = ring.tile(m);
        if (m < ntiles) {
            // pass 1: advance the state, leaving h_t in g_c's row t
            uint32_t row = tile;
            for (int q = 0; q < n; ++q, row += ROWB) {
                const int kk = __shfl_sync(kFull, kreg, q);
                float dv[NPL], bv[NPL];
                lds_own<T, NPL>(row + own_off, dv);
                lds_own<T, NPL>(row + own_off + TENS, bv);
                pd_step<NPL, LV>(h, dv, bv, pb_s, ob_s, lds_u32x2(seg_lane + kk * 256), lane, q & 1);
                stg_own<NPL>(gc + (int64_t)(t0 + q) * N, lane, h);
            }
        } else {
            // pass 2: states of this tile, hsm[q] = h_{t0+q-1}
#pragma unroll
            for (int q = 0; q <= kTS; ++q) {
                if (q > n) break;
                sts_own<NPL>(hs_lane + q * (kMaxN * 4), nst[q]);
            }
            __syncwarp();
            uint32_t row = tile + (n - 1) * ROWB;
            for (int q = n - 1; q >= 0; --q, row -= ROWB) {
                const int kk = __shfl_sync(kFull, kreg, q);
                const float gy = __shfl_sync(kFull, gyreg, q);
                float dv[NPL], cv[NPL], hq[NPL], hp[NPL], lam[NPL], gcv[NPL], gdv[NPL];
                int t4[NPL];
                lds_own<T, NPL>(row + own_off, dv);
                lds_own<T, NPL>(row + own_off + TENS, cv);
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
        if (m + kFastStages < total) {
            issue(m + kFastStages);
        }
        // the next pass-2 tile's states (written by this lane in pass 1)
        if (m + 1 >= ntiles && m + 1 < total) load_states(tile_of(m + 1));
        kreg = clamp_k(knext, K, p.status);
        gyreg = gynext;
    }
}

template <typename T, int NPL>
__global__ void __launch_bounds__(kMaxWPC * 32, 2) k_bwdC_fast(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_bc_raw[];
    unsigned char *sm_bc = smem_base256(sm_bc_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_bc, warp, lane, 4);
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    unsigned char *wbase = sm_bc + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    switch (step_variant(p.dict_stats, NPL)) {
        case 0: bwdC_fast_unit<T, NPL, 0>(p, sd, wbase, unit, lane); break;
        case 1: bwdC_fast_unit<T, NPL, 1>(p, sd, wbase, unit, lane); break;
        case 2: bwdC_fast_unit<T, NPL, 2>(p, sd, wbase, unit, lane); break;
        case 3: bwdC_fast_unit<T, NPL, 3>(p, sd, wbase, unit, lane); break;
        case kStepWin:
            if constexpr (NPL == 2) {
                bwdC_fast_unit<T, NPL, kStepWin>(p, sd, wbase, unit, lane);
                break;
            }
            [[fallthrough]];
        default: bwdC_fast_unit<T, NPL, 5>(p, sd, wbase, unit, lane); break;
    }
}

template <typename KernT>
static cudaError_t launch_bfast(KernT kern, const ChunkParams &p, size_t, cudaStream_t st) {
    return launch_units(kern, p, p.smem_per_warp, st);
}

cudaError_t launch_bwdA_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.dict_content = kDictMap;
    p.smem_per_warp = warp_smem_bytes(kFastStages, 2, (int)p.N * es);
    const size_t smem = 0;
    if (dt == PDSSM_BF16)
        return p.N == 64 ? launch_bfast(k_bwdA_fast<__nv_bfloat16, 2>, p, smem, st)
                         : launch_bfast(k_bwdA_fast<__nv_bfloat16, 1>, p, smem, st);
    return p.N == 64 ? launch_bfast(k_bwdA_fast<float, 2>, p, smem, st)
                     : launch_bfast(k_bwdA_fast<float, 1>, p, smem, st);
}

cudaError_t launch_bwdC_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.dict_content = kDictMap | kDictSeg;
    // ring, exchange buffers pb / ob and lbuf, the tile's states, barriers
    p.smem_per_warp = (kFastStages * 2 * kTS * (int)p.N * es + kBwdFastExtraFloats * 4 +
                       2 * kPbStride * 4 + kFastStages * 8 + 255) / 256 * 256;
    const size_t smem = 0;
    if (dt == PDSSM_BF16)
        return p.N == 64 ? launch_bfast(k_bwdC_fast<__nv_bfloat16, 2>, p, smem, st)
                         : launch_bfast(k_bwdC_fast<__nv_bfloat16, 1>, p, smem, st);
    return p.N == 64 ? launch_bfast(k_bwdC_fast<float, 2>, p, smem, st)
                     : launch_bfast(k_bwdC_fast<float, 1>, p, smem, st);
}

}  // namespace pdssm
