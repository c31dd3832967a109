// Device routines shared by the fast forward kernels (phases A and C in
// fwd_fast.cu) and the single-pass forward (fused.cu): phase A over one
// segment of a sequence (local readout and closed transfer) and phase C
// (carry correction in path form) over one segment, for a state that
// fills the warp (N = 32 or 64) with 16-byte aligned rows.  Written
// against explicit 32-bit shared addresses so that a step costs few
// instructions:
//   * the maps are staged with entries of the element size holding byte
//     offsets, so following a column is one shared load per step;
//   * the PD step goes through the per-map segment or window tables (or
//     the permutation step when every map is a permutation);
//   * full tiles are unrolled at compile time: row, readout and lane
//     offsets are immediates;
//   * readout partials go to the per-warp transpose buffer.
#pragma once

#include "common.cuh"
#include "transfer_ops.cuh"

namespace pdssm {

// The closed PD transfer of a segment, as the lanes hold it at the end of
// phase A: column e = lane * NPL + r moves to pos[r] / sizeof(T) with factor
// Dl[r]; v[r] is the segment's state (started from zero) at element e.
template <int NPL>
struct SegTransfer {
    int pos[NPL];
    float Dl[NPL];
    float v[NPL];
};

// Phase A over the segment of `len` steps starting at global row `row0`
// (one sequence): the local readout (when p.y is set) and the segment's
// closed transfer.  LV selects the PD step (0: the permutation step, else the
// segment-table step with LV shuffle levels).  Initialises this warp's ring
// barriers; uses tiles 0 .. ceil(len / kTS) - 1 of the ring.  Returns false
// if a staging wait gave up (status flagged, transfer undefined).
template <typename T, int NPL, int LV>
__device__ __forceinline__ bool phaseA_segment(const ChunkParams &p, const SmemDict &sd,
                                               unsigned char *wbase, int64_t row0, int len,
                                               int lane, SegTransfer<NPL> &out,
                                               const int32_t *ks = nullptr, int tbase = 0,
                                               bool init_bars = true) {
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int TENS = kTS * ROWB;
    const int K = (int)p.K;
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
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + row0 * ROWB;
    ring.src[1] = reinterpret_cast<const unsigned char *>(p.b) + row0 * ROWB;
    ring.src[2] = with_y ? reinterpret_cast<const unsigned char *>(p.c) + row0 * ROWB
                         : ring.src[1];
    if (init_bars) ring_init_bars(ring.bar0, kFastStages, lane);
    const unsigned kAll = (1u << nt) - 1u;

    const int ntiles = (len + kTS - 1) / kTS;
    for (int i = 0; i < kFastStages && i < ntiles; ++i) ring.issue_tile(tbase + i, i, kAll, lane);

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
    // selection indices: from global memory, or (ks) from this CTA's shared memory
    const int32_t *kp = ks ? ks : p.k + row0;
    auto kload = [&](int idx, bool valid) {
        return valid ? (ks ? kp[idx] : __ldg(kp + idx)) : 0;
    };
    float *yp = with_y ? p.y + row0 : nullptr;
    int kreg = clamp_k(kload(lane, lane < kTS && lane < len), K, p.status);

    for (int i = 0; i < ntiles; ++i) {
        if (!ring.wait(tbase + i)) {
            if (lane == 0) flag_status(p.status, kStTimeout);
            for (int j = i; j < ntiles && j < i + kFastStages; ++j) ring.wait(tbase + j);
            __syncwarp();
            return false;
        }
        const int t0 = i * kTS;
        const int n = min(kTS, len - t0);
        const int knext = kload(t0 + kTS + lane, lane < kTS && t0 + kTS + lane < len);
        const uint32_t row0s = ring.tile(tbase + i);
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
        if (i + kFastStages < ntiles) ring.issue_tile(tbase + i + kFastStages, i + kFastStages, kAll, lane);
        kreg = clamp_k(knext, K, p.status);
    }
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        out.pos[r] = posb[r];
        out.Dl[r] = Dl[r];
        out.v[r] = h[r];
    }
    return true;
}

// Carry correction (phase C) over the segment of `len` steps starting at
// global row `row0`, in path form: column e = lane * NPL + r of the carry
// starts with weight w[r] and follows the selected maps; y gains
// sum_e c_t[pos_t(e)] w_t(e) at every step.  The ring has NT tensors per
// stage; d goes to tensor 0 and c to tensor CQ.  Tile i of the segment uses
// ring slot tbase + i (so a warp can continue the barrier phases of an
// earlier pass over the same ring).  Returns false if a staging wait gave up.
template <typename T, int NPL, int NT, int CQ>
__device__ __forceinline__ bool phaseC_segment(const ChunkParams &p, const SmemDict &sd,
                                               uint32_t ring_s, uint32_t bar0, float *ybuf,
                                               int64_t row0, int len, float (&w)[NPL],
                                               int tbase, int lane,
                                               const int32_t *ks = nullptr) {
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int TENS = kTS * ROWB;
    const int K = (int)p.K;
    using RingT = FastRing<NT, ROWB>;
    RingT ring;
    ring.ring_s = ring_s;
    ring.bar0 = bar0;
    ring.len = len;
    ring.nt = NT;
#pragma unroll
    for (int q = 0; q < NT; ++q) ring.src[q] = reinterpret_cast<const unsigned char *>(p.d);
    ring.src[0] = reinterpret_cast<const unsigned char *>(p.d) + row0 * ROWB;
    ring.src[CQ] = reinterpret_cast<const unsigned char *>(p.c) + row0 * ROWB;
    constexpr unsigned kMask = 1u | (1u << CQ);

    const int ntiles = (len + kTS - 1) / kTS;
    for (int i = 0; i < kFastStages && i < ntiles; ++i) ring.issue_tile(tbase + i, i, kMask, lane);

    const uint32_t map_s = smem_u32(sd.map), yb_lane = smem_u32(ybuf) + lane * 4;
    constexpr int ES = (int)sizeof(T);
    int posb[NPL];   // column positions as byte offsets into a staged row
#pragma unroll
    for (int r = 0; r < NPL; ++r) posb[r] = (lane * NPL + r) * ES;
    const int32_t *kp = ks ? ks : p.k + row0;
    auto kload = [&](int idx, bool valid) {
        return valid ? (ks ? kp[idx] : __ldg(kp + idx)) : 0;
    };
    float *yp = p.y + row0;
    // the global loads of a tile (its local readout y, written by phase A,
    // and the selection indices) are issued a tile ahead of their use: y of
    // tile i + 1 and the indices of tile i + 2 load while tile i runs
    auto yload = [&](int ti) {
        const int t = ti * kTS + (lane >> 2);
        return ((lane & 3) == 0 && t < len && (lane >> 2) < kTS) ? yp[t] : 0.f;
    };
    int kreg = clamp_k(kload(lane, lane < kTS && lane < len), K, p.status);
    int knext = kload(kTS + lane, lane < kTS && kTS + lane < len);
    float ycur = yload(0);

    for (int i = 0; i < ntiles; ++i) {
        if (!ring.wait(tbase + i)) {
            if (lane == 0) flag_status(p.status, kStTimeout);
            for (int j = i; j < ntiles && j < i + kFastStages; ++j) ring.wait(tbase + j);
            __syncwarp();
            return false;
        }
        const int t0 = i * kTS;
        const int n = min(kTS, len - t0);
        const int knn = kload(t0 + 2 * kTS + lane, lane < kTS && t0 + 2 * kTS + lane < len);
        const float ynext = yload(i + 1);
        const uint32_t row0s = ring.tile(tbase + i);
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
                        acc = fmaf(lds_elem_at<T, Q * ROWB + CQ * TENS>(row0s + posb[r]), w[r], acc);
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
                    acc = fmaf(lds_elem_at<T, CQ * TENS>(row + posb[r]), w[r], acc);
                }
                sts_f32(yb, acc);
            }
        }
        warp_barrier();
        const float ys = ybuf_quad_sum(ybuf, lane);
        if ((lane & 3) == 0 && (lane >> 2) < n) yp[t0 + (lane >> 2)] = ycur + ys;
        warp_barrier();
        if (i + kFastStages < ntiles) ring.issue_tile(tbase + i + kFastStages, i + kFastStages, kMask, lane);
        kreg = clamp_k(knext, K, p.status);
        knext = knn;
        ycur = ynext;
    }
    return true;
}

}  // namespace pdssm
