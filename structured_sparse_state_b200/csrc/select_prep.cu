// Hard selection (fused logits + first argmax), dictionary preparation
// (phase A0) and index validation.
//
// Flash PD-SSM technical summary, Methodology §1: at each step the input u_t
// gives K scores through a linear map and the single highest-scoring
// dictionary matrix is used; each matrix is a one-hot column selector, held
// here as an index map pi_k : [N] -> [N] with P_k[pi_k(j), j] = 1.
#include "common.cuh"

namespace pdssm {

// ---------------------------------------------------------------------------
// k_select: one thread per (b, t) row, 128 rows per CTA.  The u tile is kept
// transposed in shared memory ([D][129] fp32, conflict-free both ways); the
// weights of one head are staged transposed ([D][KB]) and read as
// broadcasts.  Each logit is the sequential fp32 chain acc = fma(W, u, acc)
// over ascending d -- the selection contract -- so k is bit-reproducible.
// ---------------------------------------------------------------------------
constexpr int kSelRows = 128;

__host__ __device__ inline size_t sel_u_floats(int D) {
    return ((size_t)D * (kSelRows + 1) + 3) / 4 * 4;
}

template <typename TU, int KB>
__global__ void __launch_bounds__(kSelRows) k_select(const TU *__restrict__ u,
                                                     const float *__restrict__ W,
                                                     int32_t *__restrict__ k_out, int64_t rows,
                                                     int64_t L, int D, int H, int K) {
    extern __shared__ __align__(16) float sm_sel[];
    float *us = sm_sel;                          // [D][kSelRows + 1]
    // weights start on a 16-byte boundary (float4 reads) whatever D is
    float *wsm = us + sel_u_floats(D);           // [2][D][KB]
    const int tid = threadIdx.x;
    const int64_t row0 = (int64_t)blockIdx.x * kSelRows;
    const int nrows = (int)imin64(kSelRows, rows - row0);

    for (int idx = tid; idx < nrows * D; idx += kSelRows) {
        const int r = idx / D, q = idx - r * D;
        us[q * (kSelRows + 1) + r] = to_f<TU>(u[(row0 + r) * D + q]);
    }
    auto stage_w = [&](int h, float *dst) {
        for (int idx = tid; idx < D * KB; idx += kSelRows) {
            const int q = idx / KB, kk = idx - q * KB;
            dst[idx] = kk < K ? W[((int64_t)h * K + kk) * D + q] : 0.f;
        }
    };
    stage_w(0, wsm);
    __syncthreads();

    const int64_t row = row0 + tid;
    const int64_t bb = row / L, t = row - bb * L;
    for (int h = 0; h < H; ++h) {
        float *wc = wsm + (size_t)(h & 1) * D * KB;
        if (h + 1 < H) stage_w(h + 1, wsm + (size_t)((h + 1) & 1) * D * KB);
        if (tid < nrows) {
            float acc[KB];
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) acc[kk] = 0.f;
            for (int q = 0; q < D; ++q) {
                const float uq = us[q * (kSelRows + 1) + tid];
                const float4 *wr = reinterpret_cast<const float4 *>(wc + q * KB);
#pragma unroll
                for (int k4 = 0; k4 < KB / 4; ++k4) {
                    const float4 w4 = wr[k4];
                    acc[4 * k4 + 0] = __fmaf_rn(w4.x, uq, acc[4 * k4 + 0]);
                    acc[4 * k4 + 1] = __fmaf_rn(w4.y, uq, acc[4 * k4 + 1]);
                    acc[4 * k4 + 2] = __fmaf_rn(w4.z, uq, acc[4 * k4 + 2]);
                    acc[4 * k4 + 3] = __fmaf_rn(w4.w, uq, acc[4 * k4 + 3]);
                }
            }
            int best = 0;
            float bv = acc[0];
#pragma unroll
            for (int kk = 1; kk < KB; ++kk)
                if (kk < K && acc[kk] > bv) {
                    bv = acc[kk];
                    best = kk;
                }
            k_out[(bb * H + h) * L + t] = best;
        }
        __syncthreads();
    }
}

template <typename TU, int KB>
static cudaError_t select_t(const pdssm_dims &dm, const void *u, const float *W, int32_t *k_out,
                            cudaStream_t st) {
    const int64_t rows = dm.B * dm.L;
    const int D = (int)dm.D_in;
    const size_t smem = (sel_u_floats(D) + 2 * (size_t)D * KB) * sizeof(float);
    auto kern = k_select<TU, KB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (rows + kSelRows - 1) / kSelRows;
    kern<<<(unsigned)grid, kSelRows, smem, st>>>(reinterpret_cast<const TU *>(u), W, k_out,
                                                 rows, dm.L, D, (int)dm.H, (int)dm.K);
    return cudaGetLastError();
}

template <typename TU>
static cudaError_t select_k(const pdssm_dims &dm, const void *u, const float *W, int32_t *k_out,
                            cudaStream_t st) {
    if (dm.K <= 4) return select_t<TU, 4>(dm, u, W, k_out, st);
    if (dm.K <= 8) return select_t<TU, 8>(dm, u, W, k_out, st);
    if (dm.K <= 16) return select_t<TU, 16>(dm, u, W, k_out, st);
    return select_t<TU, 32>(dm, u, W, k_out, st);
}

cudaError_t launch_select(const pdssm_dims &dm, const void *u, pdssm_dtype ut, const float *W,
                          int32_t *k_out, bool use_tc, float *logits_out, float *scale_out,
                          cudaStream_t st) {
    if (dm.B * dm.L == 0) return cudaSuccess;
    if (use_tc) return launch_select_tc(dm, u, W, k_out, logits_out, scale_out, st);
    return ut == PDSSM_BF16 ? select_k<__nv_bfloat16>(dm, u, W, k_out, st)
                            : select_k<float>(dm, u, W, k_out, st);
}

// ---------------------------------------------------------------------------
// k_prep (phase A0): one warp per dictionary map.  Writes
//   * a sanitised copy of the map (entries clamped into [0, N), flagged);
//   * its slot table: tab[s][i] = the s-th source j (ascending) with
//     pi(j) = i, for s < kDcap, or kZeroSlot when i has fewer sources;
//   * its largest fan-in (the number of slots a step must visit; above kDcap
//     the kernels scan all sources instead).
// ---------------------------------------------------------------------------
constexpr int kPrepWarps = 4;

// Window table of one map with N = 64 (read by step_win, which documents the
// entry word).  Order of the segments: fan-in 8 down to 2, targets ascending
// within a fan-in, and before the first segment of an even fan-in that would
// start at an odd entry, the next single-source target (at most three such
// moves); the remaining single-source targets follow.  A segment of fan-in f
// <= 6 then reaches back at most two lanes.  dict_stats[2] gets the largest
// back-span (99 when a fan-in exceeds 8).  Lane l holds sources j = l and
// j = l + 32 (targets ta, tb, ranks rank_a, rank_b among their target's
// sources) and the fan-ins cnt0, cnt1 of targets l and l + 32; fmax is the
// map's largest fan-in.  Every index into the 64-entry scratch arrays is
// masked to stay inside them.
__device__ __forceinline__ void prep_window(int64_t m, int lane, int ta, int tb, int rank_a,
                                            int rank_b, int cnt0, int cnt1, int fmax,
                                            int *s_start, int *s_src, int *s_tgt,
                                            const int *s_cnt, int *s_ent, int *s_slot,
                                            uint2 *__restrict__ segw, int *dict_stats) {
    __syncwarp();   // the segment table's reads of the scratch arrays are done
    if (fmax > 8) {
        if (lane == 0) atomicMax(dict_stats + 2, 99);
        return;
    }
    const unsigned lt = (1u << lane) - 1u;
    // group of each fan-in: counts, and ranks of this lane's two targets
    unsigned lo[9], hi[9];
#pragma unroll
    for (int f = 1; f <= 8; ++f) {
        lo[f] = __ballot_sync(kFull, cnt0 == f);
        hi[f] = __ballot_sync(kFull, cnt1 == f);
    }
    int gstart[9];
    int ins0 = -1, ins1 = -1, ins2 = -1, nins = 0;
    const int n1 = __popc(lo[1]) + __popc(hi[1]);
    int pos = 0;
#pragma unroll
    for (int f = 8; f >= 2; --f) {
        const int nf = __popc(lo[f]) + __popc(hi[f]);
        gstart[f] = pos;
        if (nf > 0 && (f & 1) == 0 && (pos & 1) && nins < 3 && nins < n1) {
            if (nins == 0) ins0 = pos;
            else if (nins == 1) ins1 = pos;
            else ins2 = pos;
            ++nins;
            ++pos;
            gstart[f] = pos;
        }
        pos += nf * f;
    }
    const int tail = pos;
    auto start_of = [&](int f, int rank) {
        if (f == 0) return -1;
        if (f >= 2) {
            int g = 0;
#pragma unroll
            for (int q = 2; q <= 8; ++q)
                if (q == f) g = gstart[q];
            return g + rank * f;
        }
        return rank == 0 && nins > 0 ? ins0 : rank == 1 && nins > 1 ? ins1
             : rank == 2 && nins > 2 ? ins2 : tail + (rank - nins);
    };
    int r0 = 0, r1 = 0;
#pragma unroll
    for (int f = 1; f <= 8; ++f) {
        if (cnt0 == f) r0 = __popc(lo[f] & lt);
        if (cnt1 == f) r1 = __popc(lo[f]) + __popc(hi[f] & lt);
    }
    s_start[lane] = start_of(cnt0, r0);
    s_start[lane + 32] = start_of(cnt1, r1);
    __syncwarp();
    // entries of the sources j = lane, lane + 32
    const int ea = (s_start[ta & 63] + rank_a) & 63, eb = (s_start[tb & 63] + rank_b) & 63;
    s_ent[lane] = ea;
    s_ent[lane + 32] = eb;
    s_src[ea] = lane;
    s_tgt[ea] = ta;
    s_src[eb] = lane + 32;
    s_tgt[eb] = tb;
    __syncwarp();
    // bank colouring: element 2l is stored by the first store of lane l,
    // element 2l + 1 by the second; the gather of entry e is the first
    // (e even) or the second (e odd) load.  Colours 0 .. m - 1 go to the
    // elements stored first and gathered first and to those stored second
    // and gathered second, m .. 31 to the two mixed classes.
    const bool a_first = (s_ent[2 * lane] & 1) == 0, b_first = (s_ent[2 * lane + 1] & 1) == 0;
    const unsigned ma = __ballot_sync(kFull, a_first), mb = __ballot_sync(kFull, b_first);
    const int mcount = __popc(ma);
    const int col_a = a_first ? __popc(ma & lt) : mcount + __popc(~ma & lt);
    const int col_b = b_first ? mcount + __popc(mb & lt) : __popc(~mb & lt);
    s_slot[2 * lane] = col_a & 31;
    s_slot[2 * lane + 1] = 32 + (col_b & 31);
    __syncwarp();
    const int a = 2 * lane, b = 2 * lane + 1;
    const int src_a = s_src[a], src_b = s_src[b];
    const int tg_a = s_tgt[a], tg_b = s_tgt[b];
    const bool ab_same = tg_a == tg_b;
    const bool a_cont = lane > 0 && s_tgt[a - 1] == tg_a;
    const int D = a_cont ? lane - (s_start[tg_a & 63] >> 1) : 0;
    const int f0 = s_cnt[a], f1 = s_cnt[b];   // fan-ins of this lane's own targets
    const int e0 = f0 > 0 ? (s_start[a] + f0 - 1) & 63 : 0;
    const int e1 = f1 > 0 ? (s_start[b] + f1 - 1) & 63 : 0;
    const uint32_t w0 = (uint32_t)(s_slot[src_a & 63] * 4) | (uint32_t)(s_slot[src_b & 63] * 4) << 8 |
                        (uint32_t)(s_slot[a] * 4) << 16 | (uint32_t)(s_slot[b] * 4) << 24;
    const uint32_t w1 = (ab_same ? 1u : 0u) | (a_cont ? 2u : 0u) | (uint32_t)(min(D, 3)) << 2 |
                        (f0 > 0 ? 1u : 0u) << 4 | (f1 > 0 ? 1u : 0u) << 5 |
                        (uint32_t)(e0 >> 1) << 16 | (uint32_t)(e0 & 1) << 21 |
                        (uint32_t)(e1 >> 1) << 22 | (uint32_t)(e1 & 1) << 27;
    segw[m * 32 + lane] = make_uint2(w0, w1);
    const int mdw = __reduce_max_sync(kFull, D);
    if (lane == 0) atomicMax(dict_stats + 2, mdw);
}

__global__ void k_prep(const int32_t *__restrict__ pi, int64_t pi_hs, int32_t *__restrict__ dict,
                       uint2 *__restrict__ seg, uint2 *__restrict__ segw,
                       int *__restrict__ dict_stats,
                       uint8_t *__restrict__ tab, int32_t *__restrict__ fan, int64_t nmaps,
                       int K, int N, int *status) {
    __shared__ int s_off[kPrepWarps][65];   // first sorted entry of each target (+ total)
    __shared__ int s_src[kPrepWarps][64];   // sorted entries: source
    __shared__ int s_tgt[kPrepWarps][64];   // sorted entries: target
    __shared__ int s_cnt0[kPrepWarps][64];  // sources of each target among j < 32
    __shared__ int s_cnt[kPrepWarps][64];   // sources of each target
    __shared__ int s_ent[kPrepWarps][64];   // window table: entry of each source
    __shared__ int s_slot[kPrepWarps][64];  // window table: exchange slot of each element
    pdl_trigger();
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t m = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib;
    if (m >= nmaps) return;
    const int64_t dk = m / K, kk = m - dk * K;
    const int32_t *src = pi + dk * pi_hs + kk * N;
    uint8_t *t = tab + m * (kDcap * 64);
    for (int i = lane; i < kDcap * 64; i += 32) t[i] = (uint8_t)kZeroSlot;
    // the map's row, two entries per lane, sanitised once
    int ta = lane < N ? __ldg(src + lane) : 0;
    int tb = lane + 32 < N ? __ldg(src + lane + 32) : 0;
    bool bad = (lane < N && (ta < 0 || ta >= N)) || (lane + 32 < N && (tb < 0 || tb >= N));
    ta = min(max(ta, 0), N - 1);
    tb = min(max(tb, 0), N - 1);
    if (lane < N) dict[m * N + lane] = ta;
    if (lane + 32 < N) dict[m * N + lane + 32] = tb;
    __syncwarp();
    // Ranks of this lane's sources among the sources of their target
    // (ascending j): sources j = lane first, then j = lane + 32.  Lanes past N
    // carry keys no real target has.
    const unsigned lt = (1u << lane) - 1u;
    const int key_a = lane < N ? ta : 64 + lane;
    const int key_b = lane + 32 < N ? tb : 128 + lane;
    const unsigned m_a = __match_any_sync(kFull, key_a);
    const unsigned m_b = __match_any_sync(kFull, key_b);
    s_cnt0[wib][lane] = 0;
    s_cnt0[wib][lane + 32] = 0;
    s_cnt[wib][lane] = 0;
    s_cnt[wib][lane + 32] = 0;
    __syncwarp();
    if (lane < N && (m_a & lt) == 0) s_cnt0[wib][ta] = __popc(m_a);   // one writer per target
    __syncwarp();
    const int rank_a = __popc(m_a & lt);
    const int rank_b = lane + 32 < N ? s_cnt0[wib][tb] + __popc(m_b & lt) : 0;
    if (lane < N && (m_a & lt) == 0) s_cnt[wib][ta] = __popc(m_a);
    __syncwarp();
    if (lane + 32 < N && (m_b & lt) == 0) s_cnt[wib][tb] += __popc(m_b);
    __syncwarp();
    const int cnt0 = s_cnt[wib][lane], cnt1 = s_cnt[wib][lane + 32];   // fan-in of targets lane, lane + 32
    // slot tables: the r-th source of target t at t[r * 64 + t]
    if (lane < N && rank_a < kDcap) t[rank_a * 64 + ta] = (uint8_t)lane;
    if (lane + 32 < N && rank_b < kDcap) t[rank_b * 64 + tb] = (uint8_t)(lane + 32);
    // entries below each target: exclusive scan of the counts
    int inc0 = cnt0, inc1 = cnt1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y0 = __shfl_up_sync(kFull, inc0, o), y1 = __shfl_up_sync(kFull, inc1, o);
        if (lane >= o) {
            inc0 += y0;
            inc1 += y1;
        }
    }
    const int total0 = __shfl_sync(kFull, inc0, 31);
    const int below0 = inc0 - cnt0, below1 = total0 + inc1 - cnt1;
    bad = __any_sync(kFull, bad);
    if (bad && lane == 0) flag_status(status, kStBadIndex);
    const int D = __reduce_max_sync(kFull, max(cnt0, cnt1));
    if (lane == 0) {
        fan[m] = D;
        atomicMax(dict_stats + 1, D);
    }

    // segment table (fast path only: N = 32 or 64)
    if (N != 32 && N != 64) return;
    s_off[wib][lane] = below0;
    if (lane + 32 < N) s_off[wib][lane + 32] = below1;
    if (lane == 0) s_off[wib][N] = N;
    __syncwarp();
    if (lane < N) {
        const int pa = s_off[wib][ta] + rank_a;
        s_src[wib][pa] = lane;
        s_tgt[wib][pa] = ta;
    }
    if (lane + 32 < N) {
        const int pb = s_off[wib][tb] + rank_b;
        s_src[wib][pb] = lane + 32;
        s_tgt[wib][pb] = tb;
    }
    __syncwarp();
    const int npl = N / 32;
    uint32_t w0, w1;
    int dist;
    if (npl == 2) {
        const int ea = 2 * lane, eb = 2 * lane + 1;
        const int sa = s_src[wib][ea], sb = s_src[wib][eb];
        const int ga = s_tgt[wib][ea], gb = s_tgt[wib][eb];
        const bool ab_same = ga == gb;
        const bool a_cont = lane > 0 && s_tgt[wib][ea - 1] == ga;
        const bool b_end = eb + 1 >= N || s_tgt[wib][eb + 1] != gb;
        dist = lane - (s_off[wib][gb] >> 1);
        const bool has0 = s_off[wib][ea + 1] > s_off[wib][ea];
        const bool has1 = s_off[wib][eb + 1] > s_off[wib][eb];
        w0 = (uint32_t)(sa * 4) | (uint32_t)(sb * 4) << 8 | (uint32_t)(ga * 4) << 16 |
             (uint32_t)(gb * 4) << 24;
        // where this lane's own targets' sums end up: the entry that ends
        // each target's segment (lane = entry / 2; entry odd: a b entry)
        const int e0 = has0 ? s_off[wib][ea + 1] - 1 : 0;
        const int e1 = has1 ? s_off[wib][eb + 1] - 1 : 0;
        w1 = (uint32_t)dist | (ab_same ? 1u : 0u) << 8 | (a_cont ? 1u : 0u) << 9 |
             (b_end ? 1u : 0u) << 10 | (has0 ? 1u : 0u) << 11 | (has1 ? 1u : 0u) << 12 |
             (uint32_t)(e0 >> 1) << 16 | (uint32_t)(e0 & 1) << 21 | (uint32_t)(e1 >> 1) << 22 |
             (uint32_t)(e1 & 1) << 27;
    } else {
        const int e = lane;
        const int sb = s_src[wib][e], gb = s_tgt[wib][e];
        const bool b_end = e + 1 >= N || s_tgt[wib][e + 1] != gb;
        dist = lane - s_off[wib][gb];
        const bool has0 = s_off[wib][e + 1] > s_off[wib][e];
        const int e0 = has0 ? s_off[wib][e + 1] - 1 : 0;   // entry ending this lane's target
        w0 = (uint32_t)(sb * 4) << 8 | (uint32_t)(gb * 4) << 24;
        w1 = (uint32_t)dist | (b_end ? 1u : 0u) << 10 | (has0 ? 1u : 0u) << 11 |
             (uint32_t)e0 << 16 | 1u << 21;
    }
    seg[m * 32 + lane] = make_uint2(w0, w1);
    const int md = __reduce_max_sync(kFull, dist);
    if (lane == 0) atomicMax(dict_stats, md);
    if (N == 64) prep_window(m, lane, ta, tb, rank_a, rank_b, cnt0, cnt1, D, s_off[wib], s_src[wib],
                             s_tgt[wib], s_cnt[wib], s_ent[wib], s_slot[wib], segw, dict_stats);
}

cudaError_t launch_prep(const pdssm_dims &dm, const int32_t *pi, int64_t pi_hs, int32_t *dict,
                        uint2 *seg, uint2 *segw, int *dict_stats,
                        uint8_t *tab, int32_t *fan, int64_t Hd, int *status, cudaStream_t st) {
    const int64_t nmaps = Hd * dm.K;
    const int64_t grid = (nmaps + kPrepWarps - 1) / kPrepWarps;
    k_prep<<<(unsigned)grid, 32 * kPrepWarps, 0, st>>>(pi, pi_hs, dict, seg, segw, dict_stats, tab, fan,
                                                       nmaps, (int)dm.K, (int)dm.N, status);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// k_validate: counts dictionary entries outside [0, N) (counts[0]) and
// selections outside [0, K) (counts[1]).
// ---------------------------------------------------------------------------
__global__ void k_validate(const int32_t *__restrict__ pi, int64_t pi_hs, int64_t Hd, int K,
                           int N, const int32_t *__restrict__ k, int64_t nk, int *counts) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t npi = Hd * K * N;
    int bad_pi = 0, bad_k = 0;
    for (int64_t i = tid; i < npi; i += stride) {
        const int64_t dk = i / ((int64_t)K * N), rem = i - dk * K * N;
        const int v = pi[dk * pi_hs + rem];
        bad_pi += (v < 0 || v >= N);
    }
    if (k)
        for (int64_t i = tid; i < nk; i += stride) {
            const int v = k[i];
            bad_k += (v < 0 || v >= K);
        }
    if (bad_pi) atomicAdd(counts, bad_pi);
    if (bad_k) atomicAdd(counts + 1, bad_k);
}

cudaError_t launch_validate(const pdssm_dims &dm, const int32_t *pi, int64_t pi_hs,
                            const int32_t *k, int *counts, cudaStream_t st) {
    const int64_t Hd = pi_hs ? dm.H : 1;
    k_validate<<<296, 256, 0, st>>>(pi, pi_hs, Hd, (int)dm.K, (int)dm.N, k, dm.B * dm.H * dm.L,
                                    counts);
    return cudaGetLastError();
}

}  // namespace pdssm
