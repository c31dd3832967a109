// The single-pass forward (phases A, B and C in one persistent kernel,
// with the selection optionally inside it): the kernel template and its
// launcher.  Instantiated per element type and selection mode in
// fused_bf16.cu, fused_bf16_sel.cu, fused_f32.cu and fused_f32_sel.cu (so
// they compile in parallel); fused.cu dispatches and holds the
// bounded-wait self-test.
#pragma once

#include "fwd_segments.cuh"

namespace pdssm {

// ---------------------------------------------------------------------------
// Single-pass forward (phases A, B and C in one kernel).
//
// Persistent CTAs of 8 warps in teams of W warps; a team takes one chunk at
// a time, in the order of a ticket counter, chunk-major (ticket t: chunk
// t / (B H) of sequence t % (B H)), so every predecessor of a chunk in its
// sequence holds a smaller ticket and is being processed by a running team
// or is done.  The chunk is cut into W sub-chunks (W = 1 for chunks of up
// to 128 steps, else 2; see fused_warps), one per warp of the team:
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
//      scan applied to H_{c-1}) and runs phase C on its sub-chunk, reading
//      d and c again (from L2 where they are still there).
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
static __device__ __noinline__ int resolve_row(const __nv_bfloat16 *u, const float *Wsel, int D,
                                               int K, int64_t h, int64_t urow, unsigned cand) {
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
static __device__ void select_rows_mma(const ChunkParams &p, const uint32_t *Whi,
                                       const uint32_t *Wlo, float Wn, int64_t h, int64_t urow0,
                                       int n, int32_t *ks, int lane) {
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
    // fused_warps chooses 1 or 2 warps per chunk; only those are compiled
    if (W == 1) return go(k_scan_fused<T, NPL, SEL, 1>);
    return go(k_scan_fused<T, NPL, SEL, 2>);
}


// One launcher per element type and selection mode (N = 32 or 64).
cudaError_t launch_fused_bf16(ChunkParams p, cudaStream_t st);
cudaError_t launch_fused_bf16_sel(ChunkParams p, cudaStream_t st);
cudaError_t launch_fused_f32(ChunkParams p, cudaStream_t st);
cudaError_t launch_fused_f32_sel(ChunkParams p, cudaStream_t st);

}  // namespace pdssm
