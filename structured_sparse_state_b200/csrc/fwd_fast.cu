// Forward phases A and C for a state that fills the warp (N = 32 or 64) with
// 16-byte aligned rows: the arithmetic of fwd.cu, written against explicit
// 32-bit shared addresses so that a step costs few instructions:
//   * the maps are staged with entries of the element size holding byte
//     offsets, so following a column is one shared load per step;
//   * the PD step goes through the per-map segment tables (or the
//     permutation step when every map is a permutation);
//   * full tiles are unrolled at compile time: row, readout and lane offsets
//     are immediates;
//   * readout partials go to the per-warp transpose buffer.
// The general kernels in fwd.cu serve every other N and unaligned rows.
#include "common.cuh"

namespace pdssm {

// Phase A of one chunk (this warp's unit); LV selects the PD step (0: the
// permutation step, else the segment-table step with LV shuffle levels).
template <typename T, int NPL, int LV>
__device__ __forceinline__ void phaseA_fast_unit(const ChunkParams &p, const SmemDict &sd,
                                                 unsigned char *wbase, int64_t unit, int lane) {
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int TENS = kTS * ROWB;
    const int K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);
    const bool with_y = p.y != nullptr;
    const int nt = with_y ? 3 : 2;

    using RingT = FastRing<3, ROWB>;
    float *pbuf = reinterpret_cast<float *>(wbase + kFastStages * RingT::STAGEB);
    float *ybuf = pbuf + 2 * kPbStride;
    RingT ring;
    ring.ring_s = smem_u32(wbase);
    ring.bar0 = smem_u32(ybuf + kYbufFloats);
    ring.len = len;
    ring.nt = nt;
    const int64_t row0 = bh * p.L + s;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + row0 * ROWB;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.b) + row0 * ROWB;
    ring.src[2] = with_y ? reinterpret_cast<const unsigned char *>(p.c) + row0 * ROWB
                         : ring.src[1];
    ring_init_bars(ring.bar0, kFastStages, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    for (int i = 0; i < kFastStages && i < ntiles; ++i) ring.issue(i, lane);

    const uint32_t map_s = smem_u32(sd.map);
    const uint32_t seg_lane = smem_u32(sd.seg) + lane * 8;
    const uint32_t pb_s = smem_u32(pbuf), ob_s = pb_s + 256;   // both 256-byte aligned
    const uint32_t yb_lane = smem_u32(ybuf) + lane * 4;
    const uint32_t own_off = lane * NPL * (uint32_t)sizeof(T);

    constexpr int ES = (int)sizeof(T);
    float h[NPL], Dl[NPL];
    int posb[NPL];   // column positions as byte offsets into a staged row
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        h[r] = 0.f;
        Dl[r] = 1.f;
        posb[r] = (lane * NPL + r) * ES;
    }
    const int32_t *kp = p.k + row0;
    float *yp = with_y ? p.y + row0 : nullptr;
    int kreg = load_k(kp, lane, lane < kTS && lane < len, K, p.status);

    for (int i = 0; i < ntiles; ++i) {
        if (!ring.wait(i)) {
            ring.abort(i, ntiles, p.status, lane);
            return;
        }
        const int t0 = i * kTS;
        const int n = min(kTS, len - t0);
        const int knext = load_k_raw(kp, t0 + kTS + lane, lane < kTS && t0 + kTS + lane < len);
        const uint32_t row0s = ring.tile(i);
        // values of step q that do not depend on the state, loaded one step
        // ahead so their latency overlaps the previous step's work
        int kk = __shfl_sync(kFull, kreg, 0);
        uint32_t pk = map_s + kk * (N * ES);
        float dv[NPL], bv[NPL], cv[NPL];
        lds_own<T, NPL>(row0s + own_off, dv);
        lds_own<T, NPL>(row0s + own_off + TENS, bv);
        if (with_y) lds_own<T, NPL>(row0s + own_off + 2 * TENS, cv);
        uint2 e = lds_u32x2(seg_lane + kk * 256);
        // One step: transfer tracking (Delta picks up d at the column's
        // current position, then the selected map moves the column), the PD
        // step, the next step's state-independent values, the readout
        // partial.  After the last step of a tile the next-step loads read one
        // row past the tile (still inside this warp's staging area: the next
        // stage, or the buffers behind the ring) and the index held by lane n
        // (a valid map: lanes past the tile hold 0); they are never used.
        auto finish_step = [&](int q_next, const float (&dv_n)[NPL], const float (&bv_n)[NPL],
                               const float (&cv_n)[NPL], uint2 e_n, uint32_t pk_n,
                               uint32_t yb_addr) {
            if (with_y) {
                float ya = cv[0] * h[0];
#pragma unroll
                for (int r = 1; r < NPL; ++r) ya = fmaf(cv[r], h[r], ya);
                sts_f32(yb_addr, ya);
            }
            (void)q_next;
            pk = pk_n;
            e = e_n;
#pragma unroll
            for (int r = 0; r < NPL; ++r) {
                dv[r] = dv_n[r];
                bv[r] = bv_n[r];
                cv[r] = cv_n[r];
            }
        };
        if (n == kTS) {
            // full tile: steps unrolled, row and readout offsets immediate
            for_each_q(
                [&](auto qc) {
                    constexpr int Q = decltype(qc)::value;
#pragma unroll
                    for (int r = 0; r < NPL; ++r) {
                        Dl[r] *= lds_elem_at<T, Q * ROWB>(row0s + posb[r]);
                        posb[r] = lds_next_pos<T>(pk + posb[r]);
                    }
                    pd_step<NPL, LV>(h, dv, bv, pb_s, ob_s, e, lane, Q & 1);
                    const int kk_n = __shfl_sync(kFull, kreg, Q + 1);
                    float dv_n[NPL], bv_n[NPL], cv_n[NPL];
                    lds_own_at<T, NPL, (Q + 1) * ROWB>(row0s + own_off, dv_n);
                    lds_own_at<T, NPL, (Q + 1) * ROWB + TENS>(row0s + own_off, bv_n);
                    if (with_y) lds_own_at<T, NPL, (Q + 1) * ROWB + 2 * TENS>(row0s + own_off, cv_n);
                    const uint2 e_n = lds_u32x2(seg_lane + kk_n * 256);
                    finish_step(Q + 1, dv_n, bv_n, cv_n, e_n, map_s + kk_n * (N * ES),
                                yb_lane + Q * 33 * 4);
                },
                std::make_integer_sequence<int, kTS>{});
        } else {
            uint32_t row = row0s;
            for (int q = 0; q < n; ++q, row += ROWB) {
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    Dl[r] *= lds_elem_at<T, 0>(row + posb[r]);
                    posb[r] = lds_next_pos<T>(pk + posb[r]);
                }
                pd_step<NPL, LV>(h, dv, bv, pb_s, ob_s, e, lane, q & 1);
                const int kk_n = __shfl_sync(kFull, kreg, q + 1);
                const uint32_t row_n = row + ROWB;
                float dv_n[NPL], bv_n[NPL], cv_n[NPL];
                lds_own<T, NPL>(row_n + own_off, dv_n);
                lds_own<T, NPL>(row_n + own_off + TENS, bv_n);
                if (with_y) lds_own<T, NPL>(row_n + own_off + 2 * TENS, cv_n);
                const uint2 e_n = lds_u32x2(seg_lane + kk_n * 256);
                finish_step(q + 1, dv_n, bv_n, cv_n, e_n, map_s + kk_n * (N * ES),
                            yb_lane + q * 33 * 4);
            }
        }
        warp_barrier();
        if (with_y) {
            const float ys = ybuf_quad_sum(ybuf, lane);
            if ((lane & 3) == 0 && (lane >> 2) < n) yp[t0 + (lane >> 2)] = ys;
        }
        warp_barrier();
        if (i + kFastStages < ntiles) ring.issue(i + kFastStages, lane);
        kreg = clamp_k(knext, K, p.status);
    }
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e2 = lane * NPL + r;
        p.Pi[o + e2] = posb[r] / ES;
        p.Dl[o + e2] = Dl[r];
        p.v[o + e2] = h[r];
    }
}

template <typename T, int NPL>
__global__ void __launch_bounds__(kMaxWPC * 32, (sizeof(T) == 4 && NPL == 2) ? 2 : 3)
    k_phaseA_fast(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_a_raw[];
    unsigned char *sm_a = smem_base256(sm_a_raw);
    pdl_trigger();
    pdl_wait();   // the dictionary tables come from the preceding kernel
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_a, warp, lane, (int)sizeof(T));
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    unsigned char *wbase = sm_a + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    switch (step_variant(p.dict_stats)) {
        case 0: phaseA_fast_unit<T, NPL, 0>(p, sd, wbase, unit, lane); break;
        case 1: phaseA_fast_unit<T, NPL, 1>(p, sd, wbase, unit, lane); break;
        case 2: phaseA_fast_unit<T, NPL, 2>(p, sd, wbase, unit, lane); break;
        case 3: phaseA_fast_unit<T, NPL, 3>(p, sd, wbase, unit, lane); break;
        default: phaseA_fast_unit<T, NPL, 5>(p, sd, wbase, unit, lane); break;
    }
}

template <typename T, int NPL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_phaseC_fast(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_c_raw[];
    unsigned char *sm_c = smem_base256(sm_c_raw);
    pdl_trigger();
    pdl_wait();   // the carries come from the preceding kernel
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int TENS = kTS * ROWB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_c, warp, lane, (int)sizeof(T));
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int K = (int)p.K;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    if (cidx == 0 && p.h0 == nullptr) return;   // zero initial state: nothing to correct
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    unsigned char *wbase = sm_c + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    using RingT = FastRing<2, ROWB>;
    float *ybuf = reinterpret_cast<float *>(wbase + kFastStages * RingT::STAGEB);   // [kTS][33]
    RingT ring;
    ring.ring_s = smem_u32(wbase);
    ring.bar0 = smem_u32(ybuf + kYbufFloats);
    ring.len = len;
    ring.nt = 2;
    const int64_t seq_row0 = bh * p.L;
    const int64_t row0 = seq_row0 + s;
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + row0 * ROWB;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.c) + row0 * ROWB;
    ring_init_bars(ring.bar0, kFastStages, lane);

    const int ntiles = (len + kTS - 1) / kTS;
    for (int i = 0; i < kFastStages && i < ntiles; ++i) ring.issue(i, lane);

    const uint32_t map_s = smem_u32(sd.map), yb_lane = smem_u32(ybuf) + lane * 4;
    constexpr int ES = (int)sizeof(T);
    float w[NPL];
    int posb[NPL];   // column positions as byte offsets into a staged row
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        posb[r] = e * ES;
        w[r] = cidx == 0 ? p.h0[bh * p.N + e] : p.Hc[(unit - 1) * p.N + e];
    }
    const int32_t *kp = p.k + row0;
    float *yp = p.y + row0;
    int kreg = load_k(kp, lane, lane < kTS && lane < len, K, p.status);

    for (int i = 0; i < ntiles; ++i) {
        if (!ring.wait(i)) {
            ring.abort(i, ntiles, p.status, lane);
            return;
        }
        const int t0 = i * kTS;
        const int n = min(kTS, len - t0);
        const int knext = load_k_raw(kp, t0 + kTS + lane, lane < kTS && t0 + kTS + lane < len);
        const float yold = ((lane & 3) == 0 && (lane >> 2) < n) ? yp[t0 + (lane >> 2)] : 0.f;
        const uint32_t row0s = ring.tile(i);
        if (n == kTS) {
            // full tile: steps unrolled, row and readout offsets immediate
            for_each_q(
                [&](auto qc) {
                    constexpr int Q = decltype(qc)::value;
                    const int kk = __shfl_sync(kFull, kreg, Q);
                    const uint32_t pk = map_s + kk * (N * ES);
                    float acc = 0.f;
#pragma unroll
                    for (int r = 0; r < NPL; ++r) {
                        w[r] *= lds_elem_at<T, Q * ROWB>(row0s + posb[r]);
                        posb[r] = lds_next_pos<T>(pk + posb[r]);
                        acc = fmaf(lds_elem_at<T, Q * ROWB + TENS>(row0s + posb[r]), w[r], acc);
                    }
                    sts_f32_at<Q * 33 * 4>(yb_lane, acc);
                },
                std::make_integer_sequence<int, kTS>{});
        } else {
            uint32_t row = row0s;
            uint32_t yb = yb_lane;
            for (int q = 0; q < n; ++q, row += ROWB, yb += 33 * 4) {
                const int kk = __shfl_sync(kFull, kreg, q);
                const uint32_t pk = map_s + kk * (N * ES);
                float acc = 0.f;
#pragma unroll
                for (int r = 0; r < NPL; ++r) {
                    w[r] *= lds_elem_at<T, 0>(row + posb[r]);
                    posb[r] = lds_next_pos<T>(pk + posb[r]);
                    acc = fmaf(lds_elem_at<T, TENS>(row + posb[r]), w[r], acc);
                }
                sts_f32(yb, acc);
            }
        }
        warp_barrier();
        const float ys = ybuf_quad_sum(ybuf, lane);
        if ((lane & 3) == 0 && (lane >> 2) < n) yp[t0 + (lane >> 2)] = yold + ys;
        warp_barrier();
        if (i + kFastStages < ntiles) ring.issue(i + kFastStages, lane);
        kreg = clamp_k(knext, K, p.status);
    }
}

template <typename KernT>
static cudaError_t launch_fast(KernT kern, const ChunkParams &p, size_t, cudaStream_t st) {
    return launch_units(kern, p, p.smem_per_warp, st, true);
}

// The fast kernels stage with bulk copies through a two-stage ring.
bool fast_path(const ChunkParams &p) {
    return (p.N == 32 || p.N == 64) && p.bulk && p.ns == kFastStages;
}

cudaError_t launch_phaseA_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.dict_content = (dt == PDSSM_BF16 ? kDictMap16 : kDictMap) | kDictSeg;
    p.smem_per_warp = warp_smem_bytes(p.ns, 3, (int)p.N * es);
    const size_t smem = 0;
    if (dt == PDSSM_BF16)
        return p.N == 64 ? launch_fast(k_phaseA_fast<__nv_bfloat16, 2>, p, smem, st)
                         : launch_fast(k_phaseA_fast<__nv_bfloat16, 1>, p, smem, st);
    return p.N == 64 ? launch_fast(k_phaseA_fast<float, 2>, p, smem, st)
                     : launch_fast(k_phaseA_fast<float, 1>, p, smem, st);
}

cudaError_t launch_phaseC_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.dict_content = dt == PDSSM_BF16 ? kDictMap16 : kDictMap;
    // ring, readout buffer, barriers (no exchange buffers: no scatter here)
    p.smem_per_warp =
        (kFastStages * 2 * kTS * (int)p.N * es + kYbufFloats * 4 + kFastStages * 8 + 255) / 256 * 256;
    const size_t smem = 0;
    if (dt == PDSSM_BF16)
        return p.N == 64 ? launch_fast(k_phaseC_fast<__nv_bfloat16, 2>, p, smem, st)
                         : launch_fast(k_phaseC_fast<__nv_bfloat16, 1>, p, smem, st);
    return p.N == 64 ? launch_fast(k_phaseC_fast<float, 2>, p, smem, st)
                     : launch_fast(k_phaseC_fast<float, 1>, p, smem, st);
}

}  // namespace pdssm
