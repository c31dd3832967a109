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

// Phase A of one chunk (this warp's unit) for the three-phase forward: the
// transfer goes to the workspace.
template <typename T, int NPL, int LV>
__device__ __forceinline__ void phaseA_fast_unit(const ChunkParams &p, const SmemDict &sd,
                                                 unsigned char *wbase, int64_t unit, int lane) {
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);
    SegTransfer<NPL> tr;
    if (!phaseA_segment<T, NPL, LV>(p, sd, wbase, bh * p.L + s, len, lane, tr)) return;
    constexpr int ES = (int)sizeof(T);
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e2 = lane * NPL + r;
        p.Pi[o + e2] = tr.pos[r] / ES;
        p.Dl[o + e2] = tr.Dl[r];
        p.v[o + e2] = tr.v[r];
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
    switch (step_variant(p.dict_stats, NPL)) {
        case 0: phaseA_fast_unit<T, NPL, 0>(p, sd, wbase, unit, lane); break;
        case 1: phaseA_fast_unit<T, NPL, 1>(p, sd, wbase, unit, lane); break;
        case 2: phaseA_fast_unit<T, NPL, 2>(p, sd, wbase, unit, lane); break;
        case 3: phaseA_fast_unit<T, NPL, 3>(p, sd, wbase, unit, lane); break;
        case kStepWin:
            if constexpr (NPL == 2) {
                phaseA_fast_unit<T, NPL, kStepWin>(p, sd, wbase, unit, lane);
                break;
            }
            [[fallthrough]];
        default: phaseA_fast_unit<T, NPL, 5>(p, sd, wbase, unit, lane); break;
    }
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

template <typename T, int NPL>
__global__ void __launch_bounds__(kMaxWPC * 32) k_phaseC_fast(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_c_raw[];
    unsigned char *sm_c = smem_base256(sm_c_raw);
    pdl_trigger();
    pdl_wait();   // the carries come from the preceding kernel
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const SmemDict sd = stage_dict(p, sm_c, warp, lane, (int)sizeof(T));
    const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
    if (unit >= p.units) return;
    const int64_t bh = unit / p.C, cidx = unit - bh * p.C;
    if (cidx == 0 && p.h0 == nullptr) return;   // zero initial state: nothing to correct
    const int64_t s = cidx * p.chunk;
    const int len = (int)imin64(p.chunk, p.L - s);

    unsigned char *wbase = sm_c + dict_region_bytes(p) + (size_t)warp * p.smem_per_warp;
    using RingT = FastRing<2, ROWB>;
    float *ybuf = reinterpret_cast<float *>(wbase + kFastStages * RingT::STAGEB);   // [kTS][33]
    const uint32_t bar0 = smem_u32(ybuf + kYbufFloats);
    ring_init_bars(bar0, kFastStages, lane);
    float w[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        w[r] = cidx == 0 ? p.h0[bh * p.N + e] : p.Hc[(unit - 1) * p.N + e];
    }
    phaseC_segment<T, NPL, 2, 1>(p, sd, smem_u32(wbase), bar0, ybuf, bh * p.L + s, len, w, 0,
                                 lane);
}

// ---------------------------------------------------------------------------
// Single-pass forward (phases A, B and C in one kernel).
//
// Persistent CTAs of 8 warps in teams of W warps; a team takes one chunk at
// a time, in the order of a ticket counter, chunk-major (ticket t: chunk
// t / (B H) of sequence t % (B H)), so every predecessor of a chunk in its
// sequence holds a smaller ticket and is being processed by a running team
// or is done.  The chunk is cut into W sub-chunks of about 64 steps (W = 1,
// 2, 4 or 8), one per warp of the team:
//   1. each warp runs phase A on its sub-chunk (local readout into y, the
//      sub-chunk's closed transfer);
//   2. an inclusive Hillis-Steele scan over the team composes the
//      sub-chunk transfers (log2 W rounds in shared memory): warp
//      w holds T_w o ... o T_0, the last warp the chunk's transfer A_c;
//   3. the last warp publishes A_c (flag kFlagAgg); warp 0 finds the carry
//      H_{c-1} by decoupled look-back: the nearest predecessor with a
//      published carry (kFlagIncl; the sequence start counts, with h0),
//      then the aggregates of the predecessors after it applied in order;
//      it publishes H_c = A_c(H_{c-1}) (kFlagIncl) and h_last;
//   4. each warp takes its sub-chunk's carry (the exclusive prefix of the
//      scan applied to H_{c-1}) and runs phase C on its sub-chunk; d and c
//      were read a few microseconds before and are re-read from L2.
// The workspace ends up holding the same chunk transfers (Pi_c, Delta_c,
// v_c) and carries H_c as after the three-phase kernels, so the backward
// pass reads either.  Every flag wait is bounded: a chunk whose wait gives
// up flags PDSSM_ERR_TIMEOUT, takes a zero carry and still publishes, so no
// successor waits on it.
// ---------------------------------------------------------------------------
enum : int { kFlagAgg = 1, kFlagIncl = 2 };

// Transfer of chunk `unit` (as published by another CTA of this grid) in the
// layout of transfer_ops.cuh; read through L2 (__ldcg), never the
// non-coherent read-only path.
__device__ __forceinline__ void load_published(const ChunkParams &p, int64_t unit, int lane,
                                               int (&P)[2], float (&D)[2], float (&V)[2]) {
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        if (e < p.N) {
            P[r] = __ldcg(p.Pi + o + e);
            D[r] = __ldcg(p.Dl + o + e);
            V[r] = __ldcg(p.v + o + e);
        } else {
            P[r] = kPadIdx;
            D[r] = 0.f;
            V[r] = 0.f;
        }
    }
}

// Carry H_{c-1} into chunk cidx of sequence bh (warp-collective; layout of
// transfer_ops.cuh).  Each lane polls one predecessor flag; the window of 32
// moves back while every flag in it is kFlagAgg.  Returns false if the wait
// ran past p.wait_ns (x is then zero).
__device__ __forceinline__ bool lookback_carry(const ChunkParams &p, int64_t bh, int64_t cidx,
                                            bool perm, ScatterScratch &sc, int lane,
                                            float (&x)[2]) {
    const int64_t u0 = bh * p.C;
    int64_t top = cidx - 1;
    int64_t base = -1;
    bool ok = true;
    const uint64_t t0 = global_ns();
    for (;;) {
        const int64_t j = top - lane;
        // the sequence start counts as a published carry (h0)
        const int f = j >= 0 ? ld_acquire_gpu(p.look + u0 + j) : kFlagIncl;
        const unsigned incl = __ballot_sync(kFull, f >= kFlagIncl);
        const unsigned none = __ballot_sync(kFull, f < kFlagAgg);
        if (incl) {
            const int i = __ffs(incl) - 1;
            if ((none & ((1u << i) - 1u)) == 0) {
                base = top - i;
                break;
            }
        } else if (none == 0) {
            top -= 32;   // all 32 hold aggregates only: look further back
            continue;
        }
        if (global_ns() - t0 > p.wait_ns) {
            ok = false;
            break;
        }
        __nanosleep(100);
    }
    __syncwarp();
    __threadfence();
    if (!ok) {
        if (lane == 0) flag_status(p.status, kStTimeout);
        x[0] = x[1] = 0.f;
        return false;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        if (e >= p.N)
            x[r] = 0.f;
        else if (base >= 0)
            x[r] = __ldcg(p.Hc + (u0 + base) * p.N + e);
        else
            x[r] = p.h0 ? p.h0[bh * p.N + e] : 0.f;
    }
    // the aggregates after the base, oldest first; the next one's loads are
    // in flight while the current one is applied
    int P[2], Pn[2];
    float D[2], V[2], Dn[2], Vn[2];
    if (base + 1 < cidx) load_published(p, u0 + base + 1, lane, Pn, Dn, Vn);
    for (int64_t j = base + 1; j < cidx; ++j) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            P[r] = Pn[r];
            D[r] = Dn[r];
            V[r] = Vn[r];
        }
        if (j + 1 < cidx) load_published(p, u0 + j + 1, lane, Pn, Dn, Vn);
        float z[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) z[r] = D[r] * x[r];
        warp_scatter(P, z, V, x, sc, lane, perm);
    }
    return true;
}

// ---------------------------------------------------------------------------
// Hard selection inside the single-pass forward (k stays in shared memory).
// The logits of 16 rows x 16 maps per warp-level bf16 tensor-core product
// (mma m16n8k16, fp32 accumulation) against W split into W_hi = bf16(W) and
// W_lo = bf16(W - W_hi), so every product is exact and |W - W_hi - W_lo| <=
// 2^-16 |W|.  The argmax is certified as in the standalone tensor-core
// selection: with S = ||u_row|| max_k ||W_hk|| (rounded up), the product
// logit lies within (D 2^-21 + 2^-16) S of the exact sum and the contract's
// fp32 fma chain within D 2^-24 S, so the contract's first argmax is among
// the logits within twice their sum of the top one; a single candidate is
// the answer, several are decided by their exact fp32 fma chains.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Sum of squares of the two bf16 values packed in w, added to s.
__device__ __forceinline__ float sq2(uint32_t w, float s) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
    return fmaf(hi, hi, fmaf(lo, lo, s));
}

// The contract's fp32 fma chains of the candidate maps of one row (first
// maximum in ascending k).  Plain arguments: a reference to the kernel's
// parameter block would make every thread copy it to local memory.
__device__ __noinline__ int resolve_row(const __nv_bfloat16 *u, const float *Wsel, int D, int K,
                                        int64_t h, int64_t urow, unsigned cand) {
    const __nv_bfloat16 *ur = u + urow * D;
    float bv = 0.f;
    int best = -1;
    while (cand) {
        const int kk = __ffs(cand) - 1;
        cand &= cand - 1;
        const float *wr = Wsel + (h * K + kk) * D;
        float acc = 0.f;
        for (int q = 0; q < D; ++q) acc = __fmaf_rn(__ldg(wr + q), __bfloat162float(ur[q]), acc);
        if (best < 0 || acc > bv) {
            bv = acc;
            best = kk;
        }
    }
    return best;
}

// Selection of rows [0, n) starting at u row urow0 (b * L + t0) for head h:
// writes k of each row into ks[row].  Whi / Wlo: [K][D/2] packed bf16 pairs
// of this head's W; Wn = max_k ||W_hk|| rounded up.
__device__ void select_rows_mma(const ChunkParams &p, const uint32_t *Whi, const uint32_t *Wlo,
                                float Wn, int64_t h, int64_t urow0, int n, int32_t *ks, int lane) {
    const int D = p.D_in, K = (int)p.K, D2 = D / 2;
    const int g = lane >> 2, q = lane & 3;
    const float ceps = 1.01f * ((float)D * 4.76837158203125e-07f + 1.52587890625e-05f +
                                (float)D * 5.9604644775390625e-08f);
    const int ntl = K > 8 ? 2 : 1;
    for (int m0 = 0; m0 < n; m0 += 16) {
        const bool v0 = m0 + g < n, v1 = m0 + g + 8 < n;
        const uint32_t *u0 = reinterpret_cast<const uint32_t *>(
            reinterpret_cast<const __nv_bfloat16 *>(p.u) + (urow0 + m0 + g) * D);
        const uint32_t *u1 = u0 + 4 * D;   // row g + 8 (8 rows of D bf16 = 4 D words)
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float s0 = 0.f, s1 = 0.f;
        for (int kb = 0; kb < D2; kb += 8) {
            const uint32_t a0 = v0 ? __ldg(u0 + kb + q) : 0u;
            const uint32_t a1 = v1 ? __ldg(u1 + kb + q) : 0u;
            const uint32_t a2 = v0 ? __ldg(u0 + kb + q + 4) : 0u;
            const uint32_t a3 = v1 ? __ldg(u1 + kb + q + 4) : 0u;
            s0 = sq2(a2, sq2(a0, s0));
            s1 = sq2(a3, sq2(a1, s1));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                if (nt >= ntl) break;
                // rows past K (staged only for k < K) contribute zero
                const int n = nt * 8 + g;
                const int wrow = n * D2 + kb + q;
                const bool live = n < K;
                mma_bf16_16816(acc[nt], a0, a1, a2, a3, live ? Whi[wrow] : 0u,
                               live ? Whi[wrow + 4] : 0u);
                mma_bf16_16816(acc[nt], a0, a1, a2, a3, live ? Wlo[wrow] : 0u,
                               live ? Wlo[wrow + 4] : 0u);
            }
        }
        // row norms: the four lanes of a quad share rows g and g + 8
        s0 += __shfl_xor_sync(kFull, s0, 1);
        s0 += __shfl_xor_sync(kFull, s0, 2);
        s1 += __shfl_xor_sync(kFull, s1, 1);
        s1 += __shfl_xor_sync(kFull, s1, 2);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            // this lane's logits of the row: maps nt * 8 + 2 q + {0, 1}
            float lg[4];
            int kk[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    kk[nt * 2 + e] = nt * 8 + 2 * q + e;
                    lg[nt * 2 + e] = acc[nt][half * 2 + e];
                }
            float b1 = -INFINITY;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (kk[e] < K) b1 = fmaxf(b1, lg[e]);
            b1 = fmaxf(b1, __shfl_xor_sync(kFull, b1, 1));
            b1 = fmaxf(b1, __shfl_xor_sync(kFull, b1, 2));
            const float unorm = __fmul_ru(__fsqrt_ru(half ? s1 : s0), 1.0009765625f);
            const float thr = b1 - 2.0f * __fmul_ru(__fmul_ru(unorm, Wn), ceps);
            unsigned cand = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (kk[e] < K && lg[e] >= thr) cand |= 1u << kk[e];
            cand |= __shfl_xor_sync(kFull, cand, 1);
            cand |= __shfl_xor_sync(kFull, cand, 2);
            const int row = m0 + g + 8 * half;
            if (q == 0 && row < n) {
                int kv;
                if (__popc(cand) == 1) {
                    kv = __ffs(cand) - 1;
                } else {
                    // near tie, or no finite logit: the exact chains decide
                    if (cand == 0) cand = (1u << K) - 1u;
                    kv = resolve_row(reinterpret_cast<const __nv_bfloat16 *>(p.u), p.W_sel, D,
                                     K, h, urow0 + row, cand);
                }
                ks[row] = kv;
            }
        }
    }
}

// Per-warp scratch of steps 2-4, inside the warp's staging ring (idle
// between phase A and phase C): scan buffers [2][64] of P, D and V, the
// scatter scratch, and one vector for the layout change of the carry.
struct FusedScratch {
    int P[2][64];
    float D[2][64];
    float V[2][64];
    ScatterScratch sc;
    float xs[64];
};

// Persistent CTAs of kFusedCtaWarps warps, split into teams of W warps; a
// team takes one chunk (ticket) at a time and syncs on its own named
// barrier, so teams never wait for one another.  The register budget is
// sized for 24 resident warps per SM (16 for fp32 rows of 64, whose phase A
// needs more than 80 registers).
constexpr int kFusedCtaWarps = 8;

template <typename T, int NPL>
constexpr int fused_min_blocks() {
    return (sizeof(T) == 4 && NPL == 2 ? 16 : 24) / kFusedCtaWarps;
}

// Shared memory of the persistent kernel: the header (tickets, chunk states,
// carries, kFusedHeader bytes), the dictionary
// (one slot for a shared dictionary, one per team otherwise), the warps'
// regions, then (selection) each warp's indices and one staging area per
// team for W_sel's hi / lo parts.
// Header of the persistent kernel's shared memory (bytes): per team a ticket
// and the max row norm of W_sel (16 bytes), per warp its FusedChunk, per
// team the carry H_{c-1} (64 floats).
constexpr int kFusedTickets = 0;
constexpr int kFusedStates = kFusedTickets + kFusedCtaWarps * 16;
constexpr int kFusedCarries = kFusedStates + kFusedCtaWarps * 48;
constexpr int kFusedHeader = (kFusedCarries + kFusedCtaWarps * 256 + 255) / 256 * 256;

struct FusedLayout {
    size_t dict, regions, ks, wstage, total;
    int slot, smax, wbytes;
    bool wstage_own;
};
__host__ __device__ inline FusedLayout fused_layout(const ChunkParams &p, int W, bool sel) {
    FusedLayout l;
    const int teams = kFusedCtaWarps / W;
    l.slot = dict_slot_bytes((int)p.K, (int)p.N, p.dict_content);
    l.dict = (size_t)kFusedHeader;
    l.regions = l.dict + (size_t)(p.dict_hs ? teams : 1) * l.slot;
    l.ks = l.regions + (size_t)kFusedCtaWarps * p.smem_per_warp;
    l.smax = (int)((p.chunk + W - 1) / W);
    l.wbytes = 4 * (int)p.K * p.D_in;   // hi and lo bf16 parts of K rows
    // (never inside the warps' regions: their ring barriers stay live from
    // chunk to chunk)
    l.wstage_own = sel;
    l.wstage = l.ks + (sel ? (size_t)kFusedCtaWarps * l.smax * 4 : 0);
    l.total = l.wstage + (l.wstage_own ? (size_t)teams * l.wbytes : 0);
    return l;
}

__device__ __forceinline__ void team_sync(int team, int W) {
    if (W == 1)
        __syncwarp();
    else
        asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(W * 32) : "memory");
}

// Per-warp state of the chunk in progress, parked in shared memory across
// phase A so that it holds no registers there.
struct FusedChunk {
    int64_t unit, cidx, bh, row0;
    int wlen, pad;
};
static_assert(sizeof(FusedChunk) <= 48, "chunk state slot");

// Steps 2-4 of a chunk (after phase A) for one warp of a team; reloads the
// chunk's state from shared memory and advances the ring slot count tb by
// phase C's tiles.
template <typename T, int NPL, bool SEL, int W, int LV>
__device__ __forceinline__ void steps_2_to_4(const ChunkParams &p, unsigned char *sm,
                                             const SegTransfer<NPL> &tr, bool ok, int &tb) {
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int ES = (int)sizeof(T);
    using RingT = FastRing<3, ROWB>;
    constexpr bool perm = LV == 0;
    int tid = (int)threadIdx.x;
    asm volatile("" : "+r"(tid));
    const int warp = tid >> 5, lane = tid & 31;
    const int team = warp / W, tw = warp - team * W;
    const volatile FusedChunk *st = reinterpret_cast<const volatile FusedChunk *>(sm + kFusedStates) + warp;
    const int64_t unit = st->unit, cidx = st->cidx, bh = st->bh, row0 = st->row0;
    const int wlen = st->wlen;
    const FusedLayout lay = fused_layout(p, W, SEL);
    unsigned char *wteam = sm + lay.regions + (size_t)(team * W) * p.smem_per_warp;
    unsigned char *wbase = wteam + (size_t)tw * p.smem_per_warp;
    FusedScratch &fs = *reinterpret_cast<FusedScratch *>(wbase);
    FusedScratch &last = *reinterpret_cast<FusedScratch *>(wteam + (size_t)(W - 1) * p.smem_per_warp);
    float *t_carry = reinterpret_cast<float *>(sm + kFusedCarries) + team * 64;
    const int ntA = (wlen + kTS - 1) / kTS;

    // 2. the sub-chunk transfer into the scan layout, then the team scan
    __syncwarp();
#pragma unroll
    for (int r = 0; r < NPL; ++r) {
        const int e = lane * NPL + r;
        fs.P[0][e] = ok ? tr.pos[r] / ES : e;
        fs.D[0][e] = ok ? tr.Dl[r] : 1.f;
        fs.V[0][e] = ok ? tr.v[r] : 0.f;
    }
    if (NPL == 1) {   // padding elements 32 .. 63
        fs.P[0][32 + lane] = kPadIdx;
        fs.D[0][32 + lane] = 0.f;
        fs.V[0][32 + lane] = 0.f;
    }
    __syncwarp();
    Agg a;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        a.P[r] = fs.P[0][lane + 32 * r];
        a.D[r] = fs.D[0][lane + 32 * r];
        a.V[r] = fs.V[0][lane + 32 * r];
    }
    team_sync(team, W);
    int cur = 0;
#pragma unroll
    for (int dd = 1; dd < W; dd <<= 1) {
        if (tw >= dd) {
            // this warp's aggregate goes after warp (tw - dd)'s
            const FusedScratch &src =
                *reinterpret_cast<const FusedScratch *>(wbase - (size_t)dd * p.smem_per_warp);
            Agg lo;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                lo.P[r] = src.P[cur][lane + 32 * r];
                lo.D[r] = src.D[cur][lane + 32 * r];
                lo.V[r] = src.V[cur][lane + 32 * r];
            }
            compose_after(lo, fs.P[cur], fs.D[cur], a.P, a.D, a.V, fs.sc, lane, perm);
            a = lo;
        }
        const int nxt = cur ^ 1;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            fs.P[nxt][lane + 32 * r] = a.P[r];
            fs.D[nxt][lane + 32 * r] = a.D[r];
            fs.V[nxt][lane + 32 * r] = a.V[r];
        }
        cur = nxt;
        team_sync(team, W);
    }

    // 3. publish the chunk's transfer; find and publish its carry
    if (tw == W - 1) {
        const int64_t o = unit * p.N;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            if (e < p.N) {
                p.Pi[o + e] = a.P[r];
                p.Dl[o + e] = a.D[r];
                p.v[o + e] = a.V[r];
            }
        }
        if (cidx > 0) {
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_gpu(p.look + unit, kFlagAgg);
        }
    }
    if (tw == 0) {
        float x[2];
        if (cidx == 0) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int e = lane + 32 * r;
                x[r] = (p.h0 && e < p.N) ? p.h0[bh * p.N + e] : 0.f;
            }
        } else {
            lookback_carry(p, bh, cidx, perm, fs.sc, lane, x);
        }
        // H_c = A_c(H_{c-1}) with A_c from the last warp's scan buffer
        int P[2];
        float z[2], hc[2], V[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            P[r] = last.P[cur][lane + 32 * r];
            z[r] = last.D[cur][lane + 32 * r] * x[r];
            V[r] = last.V[cur][lane + 32 * r];
        }
        warp_scatter(P, z, V, hc, fs.sc, lane, perm);
        const int64_t o = unit * p.N;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int e = lane + 32 * r;
            if (e < p.N) {
                p.Hc[o + e] = hc[r];
                if (cidx == p.C - 1 && p.h_last) p.h_last[bh * p.N + e] = hc[r];
            }
            t_carry[lane + 32 * r] = e < p.N ? x[r] : 0.f;
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release_gpu(p.look + unit, kFlagIncl);
    }
    team_sync(team, W);

    // 4. this sub-chunk's carry, then its carry correction (ring slots tb ..)
    float xw[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) xw[r] = t_carry[lane + 32 * r];
    if (tw > 0) {
        const FusedScratch &prev = *reinterpret_cast<const FusedScratch *>(wbase - p.smem_per_warp);
        int P[2];
        float z[2], V[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            P[r] = prev.P[cur][lane + 32 * r];
            z[r] = prev.D[cur][lane + 32 * r] * xw[r];
            V[r] = prev.V[cur][lane + 32 * r];
        }
        warp_scatter(P, z, V, xw, fs.sc, lane, perm);
    }
    fs.xs[lane] = xw[0];
    fs.xs[lane + 32] = xw[1];
    __syncwarp();
    float w[NPL];
#pragma unroll
    for (int r = 0; r < NPL; ++r) w[r] = fs.xs[lane * NPL + r];
    // the team is done with the scratch before copies land in its rings
    fence_proxy_async_shared();
    team_sync(team, W);
    if (ok && wlen > 0 && !(cidx == 0 && tw == 0 && p.h0 == nullptr)) {
        const SmemDict sd = dict_view(p, sm + lay.dict + (p.dict_hs ? (size_t)team * lay.slot : 0));
        const int32_t *ks = SEL ? reinterpret_cast<const int32_t *>(sm + lay.ks) + warp * lay.smax
                                : nullptr;
        float *ybuf = reinterpret_cast<float *>(wbase + kFastStages * RingT::STAGEB) + 2 * kPbStride;
        phaseC_segment<T, NPL, 3, 2>(p, sd, smem_u32(wbase), smem_u32(ybuf + kYbufFloats), ybuf,
                                     row0, wlen, w, tb, lane, ks);
        tb += ntA;
    }
}

// The chunk loop of one team (every warp of the CTA runs it); LV selects
// phase A's PD step.
template <typename T, int NPL, bool SEL, int W, int LV>
__device__ __forceinline__ void fused_teams(const ChunkParams &p, unsigned char *sm) {
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int ES = (int)sizeof(T);
    using RingT = FastRing<3, ROWB>;
    constexpr bool perm = LV == 0;   // every map a permutation
    int64_t cur_head = -1;
    int tb = 0;

    for (;;) {
        // addresses are recomputed from an opaque thread index where they
        // are used, so they are not held in registers across phase A
        int tid = (int)threadIdx.x;
        asm volatile("" : "+r"(tid));
        const int warp = tid >> 5, lane = tid & 31;
        const int team = warp / W, tw = warp - team * W;
        unsigned long long *t_ticket = reinterpret_cast<unsigned long long *>(sm + kFusedTickets + team * 16);
        FusedChunk *st = reinterpret_cast<FusedChunk *>(sm + kFusedStates) + warp;
        team_sync(team, W);   // the previous chunk's reads of the header are done
        if (tw == 0 && lane == 0) {
            // after a wait gave up anywhere (status flagged), take no more
            // chunks: waits on chunks nobody will process would each run to
            // their cap
            const bool stop = (*reinterpret_cast<volatile int *>(p.status) & kStTimeout) != 0;
            *t_ticket = stop ? ~0ull : atomicAdd(p.ticket, 1ull);
        }
        team_sync(team, W);
        const int64_t tk = (int64_t)*t_ticket;
        if (tk < 0 || tk >= p.units) break;
        const FusedLayout lay = fused_layout(p, W, SEL);
        const int64_t BH = p.B * p.H;
        const int64_t cidx = tk / BH, bh = tk - cidx * BH;
        const int64_t hh = bh % p.H;
        const int64_t s0 = cidx * p.chunk;
        const int len = (int)imin64(p.chunk, p.L - s0);
        const int S = (len + W - 1) / W;
        const int ws0 = min(tw * S, len);
        const int wlen = min(S, len - ws0);
        const int64_t row0 = bh * p.L + s0 + ws0;
        if (lane == 0) {
            st->unit = bh * p.C + cidx;
            st->cidx = cidx;
            st->bh = bh;
            st->row0 = row0;
            st->wlen = wlen;
        }
        unsigned char *dict_s = sm + lay.dict + (p.dict_hs ? (size_t)team * lay.slot : 0);
        if (p.dict_hs && hh != cur_head) {
            copy_slot(dict_s, p, hh, tw * 32 + lane, W * 32, ES);
            cur_head = hh;
            team_sync(team, W);
        }
        unsigned char *wbase = sm + lay.regions + (size_t)warp * p.smem_per_warp;
        const int32_t *ks = nullptr;

        // 0. (SEL) the selection of this warp's sub-chunk, into shared memory
        if constexpr (SEL) {
            int *t_wn = reinterpret_cast<int *>(sm + kFusedTickets + team * 16 + 8);
            int32_t *ksw = reinterpret_cast<int32_t *>(sm + lay.ks) + warp * lay.smax;
            const int D = p.D_in, D2 = D / 2;
            const int64_t bb = bh / p.H;
            // W_sel of this head split into bf16 hi / lo parts in the team's
            // staging area, and max_k ||W_hk|| rounded up
            uint32_t *Whi = reinterpret_cast<uint32_t *>(sm + lay.wstage + (size_t)team * lay.wbytes);
            uint32_t *Wlo = Whi + (int)p.K * D2;
            if (tw == 0 && lane == 0) *t_wn = 0;
            team_sync(team, W);
            for (int rr = tw; rr < (int)p.K; rr += W) {
                float ss = 0.f;
                for (int d2 = lane; d2 < D2; d2 += 32) {
                    const float2 wv = *reinterpret_cast<const float2 *>(
                        p.W_sel + (hh * p.K + rr) * D + 2 * d2);
                    const float w0 = wv.x, w1 = wv.y;
                    const __nv_bfloat16 h0b = __float2bfloat16_rn(w0), h1b = __float2bfloat16_rn(w1);
                    const __nv_bfloat16 l0b = __float2bfloat16_rn(w0 - __bfloat162float(h0b));
                    const __nv_bfloat16 l1b = __float2bfloat16_rn(w1 - __bfloat162float(h1b));
                    Whi[rr * D2 + d2] = (uint32_t)__bfloat16_as_ushort(h0b) |
                                        ((uint32_t)__bfloat16_as_ushort(h1b) << 16);
                    Wlo[rr * D2 + d2] = (uint32_t)__bfloat16_as_ushort(l0b) |
                                        ((uint32_t)__bfloat16_as_ushort(l1b) << 16);
                    ss = __fmaf_ru(w0, w0, ss);
                    ss = __fmaf_ru(w1, w1, ss);
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) ss = __fadd_ru(ss, __shfl_xor_sync(kFull, ss, o));
                if (lane == 0) atomicMax(t_wn, __float_as_int(ss));   // non-negative: bits order
            }
            team_sync(team, W);
            const float Wn = __fmul_ru(__fsqrt_ru(__int_as_float(*t_wn)), 1.0009765625f);
            select_rows_mma(p, Whi, Wlo, Wn, hh, bb * p.L + s0 + ws0, wlen, ksw, lane);
            __syncwarp();
            if (p.k_out)
                for (int i = lane; i < wlen; i += 32) p.k_out[row0 + i] = ksw[i];
            ks = ksw;
            // the team is done with W_sel before phase A's copies land
            fence_proxy_async_shared();
            team_sync(team, W);
        }

        // 1. phase A of this warp's sub-chunk (ring slots tb ..)
        SegTransfer<NPL> tr;
        const bool ok =
            phaseA_segment<T, NPL, LV>(p, dict_view(p, dict_s), wbase, row0, wlen, lane, tr, ks, tb, false);
        tb += (wlen + kTS - 1) / kTS;
        steps_2_to_4<T, NPL, SEL, W, LV>(p, sm, tr, ok, tb);
    }
}

template <typename T, int NPL, bool SEL, int W>
__global__ void __launch_bounds__(kFusedCtaWarps * 32, (fused_min_blocks<T, NPL>()))
    k_scan_fused(const ChunkParams p) {
    extern __shared__ __align__(128) unsigned char sm_f_raw[];
    unsigned char *sm = smem_base256(sm_f_raw);
    pdl_trigger();
    pdl_wait();   // dictionary tables and cleared flags come from the preceding work
    constexpr int N = 32 * NPL;
    constexpr int ROWB = N * (int)sizeof(T);
    constexpr int ES = (int)sizeof(T);
    using RingT = FastRing<3, ROWB>;
    static_assert(kFastStages * RingT::STAGEB >= (int)sizeof(FusedScratch),
                  "scan scratch must fit the staging ring");
    const FusedLayout lay = fused_layout(p, W, SEL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int team = warp / W;
    unsigned char *dict_s = sm + lay.dict + (p.dict_hs ? (size_t)team * lay.slot : 0);
    unsigned char *wbase = sm + lay.regions + (size_t)warp * p.smem_per_warp;
    float *ybuf = reinterpret_cast<float *>(wbase + kFastStages * RingT::STAGEB) + 2 * kPbStride;
    const uint32_t bar0 = smem_u32(ybuf + kYbufFloats);
    // a shared dictionary is staged once; this warp's ring barriers start
    // here and keep their phases from chunk to chunk (slot tb)
    if (p.dict_hs == 0) copy_slot(dict_s, p, 0, threadIdx.x, blockDim.x, ES);
    ring_init_bars(bar0, kFastStages, lane);
    __syncthreads();
    switch (step_variant(p.dict_stats, NPL)) {
        case 0: fused_teams<T, NPL, SEL, W, 0>(p, sm); break;
        case 1: fused_teams<T, NPL, SEL, W, 1>(p, sm); break;
        case 2: fused_teams<T, NPL, SEL, W, 2>(p, sm); break;
        case 3: fused_teams<T, NPL, SEL, W, 3>(p, sm); break;
        case kStepWin:
            if constexpr (NPL == 2) {
                fused_teams<T, NPL, SEL, W, kStepWin>(p, sm);
                break;
            }
            [[fallthrough]];
        default: fused_teams<T, NPL, SEL, W, 5>(p, sm); break;
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

// Self-test of the bounded waits (a failure made on purpose, without a
// fault): which = 0 runs the look-back of chunk 1 of a sequence whose chunk 0
// never publishes; which = 1 waits on an mbarrier that nothing completes.
// Either gives up after p.wait_ns and flags PDSSM_ERR_TIMEOUT.  One warp.
__global__ void k_wait_selftest(const ChunkParams p, int which) {
    __shared__ __align__(16) ScatterScratch sc;
    __shared__ __align__(8) uint64_t bar;
    const int lane = threadIdx.x & 31;
    if (which == 0) {
        float x[2];
        lookback_carry(p, 0, 1, true, sc, lane, x);
    } else {
        if (lane == 0) {
            mbar_init(smem_u32(&bar), 1);
            fence_mbar_init();
        }
        __syncwarp();
        const bool done = mbar_wait_bounded(smem_u32(&bar), 0, p.wait_ns);
        if (!done && lane == 0) flag_status(p.status, kStTimeout);
    }
}

cudaError_t launch_wait_selftest(const ChunkParams &p, int which, cudaStream_t st) {
    k_wait_selftest<<<1, 32, 0, st>>>(p, which);
    return cudaGetLastError();
}

// The single-pass forward serves the fast-path shapes (one CTA per chunk:
// the grid must fit the launch limit).
bool fused_path(const ChunkParams &p) { return fast_path(p) && p.units <= 0x7fffffff; }

// The selection runs inside the single-pass forward for bf16 u with D_in a
// multiple of 16 (at most 256), K <= 16, and chunks of at most 1024 steps
// (their indices stay in shared memory).
bool fused_select_ok(const ChunkParams &p, const void *u, const float *W) {
    return fused_path(p) && p.D_in % 16 == 0 && p.D_in >= 16 && p.D_in <= 256 && p.K <= 16 &&
           p.chunk <= 1024 && ((uintptr_t)u % 16) == 0 && ((uintptr_t)W % 16) == 0;
}

// Warps (sub-chunks) per chunk of the single-pass forward, by measurement on
// the three benchmark workloads (chunk 128: 1 warp per chunk; chunk 256: 2).
// More warps per chunk shorten the distance between phase A's read of a
// sub-chunk and phase C's re-read (more L2 hits) but add team barriers and a
// scan per chunk, which cost more than the hits save.
static int fused_warps(int64_t chunk) { return chunk <= 128 ? 1 : 2; }

// The single-pass forward: persistent CTAs (as many as fit the GPU, at most
// one team per chunk), each of teams of fused_warps(chunk) warps; with
// `select`, a team also takes its chunk's selection (p.u, p.W_sel).
template <typename T, int NPL, bool SEL>
static cudaError_t launch_fused_t(ChunkParams p, cudaStream_t st) {
    const int W = fused_warps(p.chunk);
    p.wpc = kFusedCtaWarps;
    const size_t smem = fused_layout(p, W, SEL).total + 256;
    auto go = [&](auto kern) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 0, per_sm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedCtaWarps * 32,
                                                               smem)) != cudaSuccess)
            return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        const int64_t teams = kFusedCtaWarps / W;
        const int64_t need = (p.units + teams - 1) / teams;
        const int64_t grid = imin64((int64_t)sms * per_sm, need);
        return launch_pdl(kern, dim3((unsigned)grid), dim3(kFusedCtaWarps * 32), smem, st, p);
    };
    switch (W) {
        case 1: return go(k_scan_fused<T, NPL, SEL, 1>);
        case 2: return go(k_scan_fused<T, NPL, SEL, 2>);
        case 4: return go(k_scan_fused<T, NPL, SEL, 4>);
        default: return go(k_scan_fused<T, NPL, SEL, 8>);
    }
}

cudaError_t launch_scan_fused(ChunkParams p, pdssm_dtype dt, cudaStream_t st, bool select) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.dict_content = (dt == PDSSM_BF16 ? kDictMap16 : kDictMap) | kDictSeg;
    p.smem_per_warp = warp_smem_bytes(kFastStages, 3, (int)p.N * es);
    if (select) {
        if (dt == PDSSM_BF16)
            return p.N == 64 ? launch_fused_t<__nv_bfloat16, 2, true>(p, st)
                             : launch_fused_t<__nv_bfloat16, 1, true>(p, st);
        return p.N == 64 ? launch_fused_t<float, 2, true>(p, st)
                         : launch_fused_t<float, 1, true>(p, st);
    }
    if (dt == PDSSM_BF16)
        return p.N == 64 ? launch_fused_t<__nv_bfloat16, 2, false>(p, st)
                         : launch_fused_t<__nv_bfloat16, 1, false>(p, st);
    return p.N == 64 ? launch_fused_t<float, 2, false>(p, st) : launch_fused_t<float, 1, false>(p, st);
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
