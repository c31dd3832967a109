// Warp-level operations on closed PD transfers (Pi, Delta, v) of N <= 64
// elements: the arbitrary-fan-in scatter x -> P_Pi diag(Delta) x + v and the
// composition of two transfers.  Used by the carry scan (phase B) and by the
// single-pass forward's in-CTA scan and look-back.
//
// Element layout inside a warp: lane l holds elements j = l and j = l + 32
// (slot 1 is padding when N <= 32).  Padding elements carry index 63, factor
// 0 and offset 0; with N < 64 no real index reaches 63, and with N = 64 there
// is no padding, so padding never touches a stored entry.
#pragma once

#include "common.cuh"

namespace pdssm {

constexpr int kPadIdx = 63;

// Per-warp scratch of the scatter (64 entries each).
struct ScatterScratch {
    int cnt[64];
    int off[64];
    int key[64];
    float val[64];
    float sum[64];
};

// out[i] = V[i] + sum_{j : P[j] = i} Z[j] over the warp's 64 elements, for an
// arbitrary index map (maps composed over a chunk often send most columns to
// one target, so no bounded fan-in is assumed).  Deterministic either way:
// a small image sums each target by a warp butterfly; otherwise the entries
// are sorted by target (ascending j within a target, by counting ranks) and
// each target's entries are summed by a segmented scan over the sorted
// order.  The trees of additions depend only on the map.
__device__ __forceinline__ void warp_scatter(const int (&P)[2], const float (&Z)[2],
                                             const float (&V)[2], float (&out)[2],
                                             ScatterScratch &sc, int lane, bool perm) {
    if (perm) {
        // every map is a permutation, so composed maps are too: each target
        // has one source (padding entries all write 0 to index 63, which no
        // real target uses when N < 64, and N = 64 has no padding)
        sc.val[P[0]] = Z[0];
        sc.val[P[1]] = Z[1];
        __syncwarp();
        out[0] = sc.val[lane] + V[0];
        out[1] = sc.val[lane + 32] + V[1];
        __syncwarp();
        return;
    }
    {
        // Maps composed over whole chunks usually send all columns to one or
        // two targets: for up to kSmallImage distinct targets, each target's
        // sum is a warp butterfly over the entries aimed at it (smallest
        // target first).  A larger image falls through to the sort below.
        constexpr int kSmallImage = 4;
        bool p0 = true, p1 = true;   // entries not yet summed
        float s0 = 0.f, s1 = 0.f;   // sums of this lane's own targets lane, lane + 32
        bool got0 = false, got1 = false;
        for (int round = 0; round < kSmallImage; ++round) {
            const unsigned key = min(p0 ? (unsigned)P[0] : 0xffffu, p1 ? (unsigned)P[1] : 0xffffu);
            const unsigned t = __reduce_min_sync(kFull, key);
            if (t == 0xffffu) break;
            float c = (p0 && (unsigned)P[0] == t) ? Z[0] : 0.f;
            if (p1 && (unsigned)P[1] == t) c += Z[1];
#pragma unroll
            for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
            if ((int)(t & 31u) == lane) {
                if (t < 32u) {
                    s0 = c;
                    got0 = true;
                } else {
                    s1 = c;
                    got1 = true;
                }
            }
            p0 = p0 && (unsigned)P[0] != t;
            p1 = p1 && (unsigned)P[1] != t;
        }
        if (!__any_sync(kFull, p0 || p1)) {
            out[0] = (got0 ? s0 : 0.f) + V[0];
            out[1] = (got1 ? s1 : 0.f) + V[1];
            return;
        }
    }
    const unsigned lt = (1u << lane) - 1u;
    const unsigned m0 = __match_any_sync(kFull, P[0]);
    const unsigned m1 = __match_any_sync(kFull, P[1]);
    const int r0 = __popc(m0 & lt), r1 = __popc(m1 & lt);
    sc.cnt[lane] = 0;
    sc.cnt[lane + 32] = 0;
    __syncwarp();
    if (r0 == 0) sc.cnt[P[0]] = __popc(m0);   // one writer per index
    __syncwarp();
    const int rank1 = sc.cnt[P[1]] + r1;       // slot-1 entries follow slot-0 ones
    __syncwarp();
    if (r1 == 0) sc.cnt[P[1]] += __popc(m1);
    __syncwarp();
    // exclusive scan of the 64 counts, bins 2 l and 2 l + 1 per lane
    const int c0 = sc.cnt[2 * lane], c1 = sc.cnt[2 * lane + 1];
    int incl = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
    }
    const int ex = incl - c0 - c1;
    sc.off[2 * lane] = ex;
    sc.off[2 * lane + 1] = ex + c0;
    __syncwarp();
    const int pos0 = sc.off[P[0]] + r0, pos1 = sc.off[P[1]] + rank1;
    sc.key[pos0] = P[0];
    sc.val[pos0] = Z[0];
    sc.key[pos1] = P[1];
    sc.val[pos1] = Z[1];
    __syncwarp();
    // segmented inclusive scan over sorted entries 2 l, 2 l + 1
    const int ka = sc.key[2 * lane], kb = sc.key[2 * lane + 1];
    const float za = sc.val[2 * lane], zb = sc.val[2 * lane + 1];
    const int kprev = __shfl_up_sync(kFull, kb, 1);     // entry 2 l - 1
    const int knext = __shfl_down_sync(kFull, ka, 1);   // entry 2 l + 2
    const bool joins_left = lane > 0 && kprev == ka;    // entry 2 l continues a segment
    float sv = ka == kb ? za + zb : zb;
    int sf = (ka != kb || !joins_left) ? 1 : 0;          // segment of 2 l + 1 starts here
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float yv = __shfl_up_sync(kFull, sv, o);
        const int yf = __shfl_up_sync(kFull, sf, o);
        if (lane >= o && !sf) {
            sv = yv + sv;
            sf = yf;
        }
    }
    const float sprev = __shfl_up_sync(kFull, sv, 1);
    if (ka != kb) sc.sum[ka] = joins_left ? sprev + za : za;   // entry 2 l ends a segment
    if (lane == 31 || knext != kb) sc.sum[kb] = sv;          // entry 2 l + 1 ends a segment
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = lane + 32 * r;
        out[r] = sc.cnt[i] > 0 ? sc.sum[i] + V[r] : V[r];
    }
    __syncwarp();
}

// Chunk transfer `unit` in the phase-B layout.
__device__ __forceinline__ void load_transfer2(const ChunkParams &p, int64_t unit, int lane,
                                               int (&P)[2], float (&D)[2], float (&V)[2]) {
    const int64_t o = unit * p.N;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int e = lane + 32 * r;
        if (e < p.N) {
            P[r] = __ldg(p.Pi + o + e);
            D[r] = __ldg(p.Dl + o + e);
            V[r] = __ldg(p.v + o + e);
        } else {
            P[r] = kPadIdx;
            D[r] = 0.f;
            V[r] = 0.f;
        }
    }
}

// Aggregate (P, D, V) of a run of chunks in one warp, laid out as above.
struct Agg {
    int P[2];
    float D[2], V[2];
};

// a <- T o a (a first, then T), where T's index map and factors are staged
// in shared memory (tP, tD) for the gathers and (TP, TD, TV) are this lane's
// entries of T.
__device__ __forceinline__ void compose_after(Agg &a, const int *tP, const float *tD,
                                              const int (&TP)[2], const float (&TD)[2],
                                              const float (&TV)[2], ScatterScratch &sc,
                                              int lane, bool perm) {
    float z[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) z[r] = TD[r] * a.V[r];
    float nv[2];
    warp_scatter(TP, z, TV, nv, sc, lane, perm);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int q = a.P[r];
        a.D[r] = a.D[r] * tD[q];
        a.P[r] = tP[q];
        a.V[r] = nv[r];
    }
}

}  // namespace pdssm
