// Hard selection on the 5th-generation tensor cores (tcgen05), exact under
// the fp32 fma-chain contract of pdssm_select.
//
// Flash PD-SSM technical summary, Methodology §1: the scores of step t are a
// linear map of u_t and the argmax picks the dictionary entry.  The scores of
// all heads for a tile of 128 rows (b, t) form one dense product
//   logits[128 x H*K] = u[128 x D] * W^T[D x H*K],
// which runs as tcgen05.mma (kind::f16, bf16 operands, fp32 accumulators in
// tensor memory).  W (fp32) is split into W_hi = bf16(W) and
// W_lo = bf16(W - W_hi); u must be bf16, so every product is exact and
// |W - W_hi - W_lo| <= 2^-16 |W|.
//
// Certification.  Let S = ||u_row||_2 * max_k ||W_hk||_2 >= sum_d |u_d W_kd|
// (Cauchy-Schwarz).  The tensor-core logit differs from the exact real sum
// by at most (D * 2^-21 + 2^-16) S (the first term allows each of the 2D
// products to lose 2 ulp of fp32 in the accumulation), and the contract's
// fp32 fma chain differs from it by at most D * 2^-24 S.  With eps the sum of
// both, any k whose tensor-core logit is below top-1 minus 2 eps has an fma
// logit strictly below the fma logit of top-1, so the contract's first
// argmax is among the candidates within 2 eps of the top.  One candidate:
// it is the answer.  Several: the epilogue evaluates their fp32 fma chains
// exactly and takes the first maximum, so k is bit-for-bit the contract's
// result either way.
//
// Operand layouts in shared memory (K-major), chosen by D:
//   D a multiple of 64: 128-byte swizzle.  A: [D/64 atoms][128 rows][128 B]
//     (TMA boxes of 64 x 128 with the 128-byte swizzle); B likewise with NP
//     rows per atom and part.  8-row groups are 1024 bytes apart; a k-step
//     of 16 moves 32 bytes inside an atom row.
//   otherwise, no swizzle, 16-byte core rows.  A: [D/8 chunks][128 rows][16 B]
//     (TMA boxes of 8 x 128); B: [2 parts][D/8 chunks][NP rows][16 B]; a
//     k-step covers two chunks (leading byte offset = one chunk slab) and
//     rows advance by 16 bytes (stride byte offset = 128 bytes per 8 rows).
// NP = H*K rounded up to 16.
//
// Pipeline (one persistent CTA per SM): warp 16 (one thread) issues the TMA
// copies of u tiles into a two-stage ring and the MMAs into two TMEM
// accumulators; warps 0-15 read the row norms from the staged tile, then the
// finished accumulator, and decide.  mbarriers hand the stages over: a tile
// stage is free once its product is done and the epilogue has read its
// norms; an accumulator is free once the epilogue has read it.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace pdssm {

constexpr int kTcRows = 128;
constexpr int kTcEpiWarps = 16;                   // four per group of 32 TMEM lanes
constexpr int kTcThreads = (kTcEpiWarps + 1) * 32;   // + one control warp

// Shared-memory matrix descriptor of tcgen05.mma: start address, leading and
// stride byte offsets (16-byte units), descriptor version 1 (sm_100), base
// offset 0, layout type 0 (no swizzle) or 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                                   bool sw128) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    if (sw128) d |= (uint64_t)2 << 61;
    return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
// K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kTcRows >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u),
        "r"(0u), "r"(0u)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

struct TcSelectParams {
    const float *W;          // [H][K][D] fp32
    const __nv_bfloat16 *u;  // [rows][D]
    int32_t *k_out;          // [B][H][L]
    float *logits_out;       // test hook: raw tensor-core logits [rows][H*K], or NULL
    float *scale_out;        // test hook: ||u_row|| * max_k ||W_hk|| (rounded up) [rows][H]
    int64_t rows, L;
    int D, H, K, NP;         // NP = H*K rounded up to 16
    int ntiles;
    uint32_t tcols;          // TMEM columns per accumulator: NP rounded up to a power of 2 >= 32
};

// Near ties wait in a per-warp queue and are resolved lane-parallel.
struct TieJob {
    int64_t row;
    int h;
    unsigned cand;
};
constexpr int kTieQ = 64;   // entries per warp; flushed when 32 more might not fit

// Dynamic shared memory (1024-byte aligned): [B parts][A x 2]
// [row-norm partials 2 x 4 x 128][tie queues][tie counts][Wn H floats]
// [8 barriers][tmem slot]
__host__ __device__ inline size_t tc_b_bytes(int D, int NP) { return (size_t)2 * D * NP * 2; }
__host__ __device__ inline size_t tc_a_bytes(int D) { return (size_t)kTcRows * D * 2; }
constexpr size_t kTcNormBytes = (size_t)2 * 4 * kTcRows * 4;
constexpr size_t kTcTieBytes = (size_t)kTcEpiWarps * kTieQ * sizeof(TieJob) + 64;
__host__ __device__ inline size_t tc_smem_bytes(int D, int NP, int H) {
    return 1024 + tc_b_bytes(D, NP) + 2 * tc_a_bytes(D) + kTcNormBytes + kTcTieBytes +
           ((size_t)H * 4 + 15) / 16 * 16 + 128;
}

// Byte offset of element (n, d) of a K-major operand with `rows` rows.
template <bool SW>
__device__ __forceinline__ uint32_t tc_elem_off(int n, int d, int rows) {
    if constexpr (SW) {
        const int c = (d & 63) >> 3;
        return (uint32_t)((d >> 6) * rows * 128 + n * 128 + ((c ^ (n & 7)) << 4) + (d & 7) * 2);
    } else {
        return (uint32_t)(((d >> 3) * rows + n) * 16 + (d & 7) * 2);
    }
}

template <int KT, bool SW>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_select_tc(const __grid_constant__ CUtensorMap umap, const TcSelectParams p) {
    extern __shared__ __align__(1024) unsigned char sm_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    pdl_trigger();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int D = p.D, NP = p.NP, H = p.H, K = KT;
    const int nkc = D / 8;
    unsigned char *Bs = sm;                               // [2 parts] operand B
    unsigned char *As = Bs + tc_b_bytes(D, NP);           // [2 stages] operand A
    float *npart = reinterpret_cast<float *>(As + 2 * tc_a_bytes(D));   // [2][4 parts][128]
    TieJob *tieq = reinterpret_cast<TieJob *>(reinterpret_cast<unsigned char *>(npart) + kTcNormBytes);
    int *tiecnt = reinterpret_cast<int *>(tieq + kTcEpiWarps * kTieQ);
    float *Wn = reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(npart) + kTcNormBytes +
                                          kTcTieBytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<unsigned char *>(Wn) +
                                                  ((size_t)H * 4 + 15) / 16 * 16);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
    // a_full[2]: tile landed; a_empty[2]: tile consumed (MMA done + norms
    // read); t_full[2]: accumulator ready; t_empty[2]: accumulator read
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    const int A_FULL = 0, A_EMPTY = 2, T_FULL = 4, T_EMPTY = 6;

    const uint32_t abytes = (uint32_t)tc_a_bytes(D);
    auto issue_a = [&](int tile, int stage) {
        const uint32_t b = bar(A_FULL + stage);
        mbar_expect_tx(b, abytes);
        const uint32_t dst = smem_u32(As + (size_t)stage * abytes);
        if constexpr (SW) {
            for (int q = 0; q < D / 64; ++q)
                tma_load_2d(dst + q * (kTcRows * 128), &umap, q * 64, tile * kTcRows, b);
        } else {
            for (int q = 0; q < nkc; ++q)
                tma_load_2d(dst + q * (kTcRows * 16), &umap, q * 8, tile * kTcRows, b);
        }
    };
    // barriers first, so the first tiles' copies overlap the weight split
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(A_FULL + s), 1);
            mbar_init(bar(A_EMPTY + s), 1 + kTcEpiWarps);
            mbar_init(bar(T_FULL + s), 1);
            mbar_init(bar(T_EMPTY + s), kTcEpiWarps);
        }
        fence_mbar_init();
        for (int s = 0; s < 2; ++s)
            if ((int)blockIdx.x + s * (int)gridDim.x < p.ntiles)
                issue_a(blockIdx.x + s * gridDim.x, s);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(2u * p.tcols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int h = tid; h < H; h += kTcThreads) Wn[h] = 0.f;
    if (tid < kTcEpiWarps) tiecnt[tid] = 0;
    __syncthreads();

    // ---- weights: split into hi/lo bf16 parts.  One warp per row n of W
    // (rows past H*K are zero), four consecutive d per lane, eight rows per
    // pass so their loads are in flight together.  The squared row norm
    // (rounded up) goes to the head's maximum.
    const int HK = H * K;
    constexpr int kRowsPerPass = 8;
    constexpr int kWarps = kTcThreads / 32;
    const size_t part_bytes = (size_t)D * NP * 2;
    for (int n0 = warp; n0 < NP; n0 += kRowsPerPass * kWarps) {
        float ss[kRowsPerPass];
#pragma unroll
        for (int j = 0; j < kRowsPerPass; ++j) ss[j] = 0.f;
        for (int d0 = lane * 4; d0 < D; d0 += 128) {
            float4 w[kRowsPerPass];
#pragma unroll
            for (int j = 0; j < kRowsPerPass; ++j) {
                const int n = n0 + j * kWarps;
                w[j] = n < HK ? __ldg(reinterpret_cast<const float4 *>(p.W + (int64_t)n * D + d0))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int j = 0; j < kRowsPerPass; ++j) {
                const int n = n0 + j * kWarps;
                if (n >= NP) continue;
                const float wv[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
                __nv_bfloat16 hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    hi[e] = __float2bfloat16_rn(wv[e]);
                    lo[e] = __float2bfloat16_rn(wv[e] - __bfloat162float(hi[e]));
                    ss[j] = __fmaf_ru(wv[e], wv[e], ss[j]);
                }
                const uint32_t off = tc_elem_off<SW>(n, d0, NP);
                *reinterpret_cast<uint2 *>(Bs + off) = *reinterpret_cast<const uint2 *>(hi);
                *reinterpret_cast<uint2 *>(Bs + part_bytes + off) =
                    *reinterpret_cast<const uint2 *>(lo);
            }
        }
#pragma unroll
        for (int j = 0; j < kRowsPerPass; ++j) {
#pragma unroll
            for (int o = 16; o; o >>= 1) ss[j] = __fadd_ru(ss[j], __shfl_xor_sync(kFull, ss[j], o));
            const int n = n0 + j * kWarps;
            // non-negative floats order like their bit patterns
            if (lane == 0 && n < HK) atomicMax(reinterpret_cast<int *>(Wn + n / K), __float_as_int(ss[j]));
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    // per-head bound on ||W_hk||_2 (rounded up)
    for (int h = tid; h < H; h += kTcThreads) Wn[h] = __fmul_ru(__fsqrt_ru(Wn[h]), 1.0009765625f);
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tcols = p.tcols;

    // The weight split and the first copies of u (inputs) may overlap the
    // preceding kernel; k_out, which it may still read, is written only after
    // it has completed.
    pdl_wait();
    bool ok = true;
    if (warp == kTcEpiWarps) {
        // ---- control: the copy of tile j + 1 into the stage tile j - 1 used
        // (as soon as that stage is free: its product done and its norms
        // read), then the MMAs of tile j
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(NP);
            const uint32_t bbase = smem_u32(Bs);
            int j = 0;
            for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++j) {
                const int s = j & 1;
                // tile j + 1 goes to the stage of tile j - 1 (the first two
                // tiles were issued before the weight split)
                const int next = tile + gridDim.x;
                if (j >= 1 && next < p.ntiles) {
                    const int sp = s ^ 1;
                    ok = mbar_wait_bounded(bar(A_EMPTY + sp), (uint32_t)(((j - 1) >> 1) & 1)) && ok;
                    issue_a(next, sp);
                }
                ok = mbar_wait_bounded(bar(A_FULL + s), (uint32_t)((j >> 1) & 1)) && ok;
                if (j >= 2)
                    ok = mbar_wait_bounded(bar(T_EMPTY + s), (uint32_t)(((j - 2) >> 1) & 1)) && ok;
                tc_fence_after();
                const uint32_t abase = smem_u32(As + (size_t)s * abytes);
                const uint32_t dacc = tmem + (uint32_t)s * tcols;
                int acc = 0;
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint64_t ad;
                    uint32_t boff;
                    if constexpr (SW) {
                        const uint32_t koff = (uint32_t)((ks >> 2) * kTcRows * 128 + (ks & 3) * 32);
                        ad = umma_smem_desc(abase + koff, 16, 1024, true);
                        boff = (uint32_t)((ks >> 2) * NP * 128 + (ks & 3) * 32);
                    } else {
                        ad = umma_smem_desc(abase + 2 * ks * (kTcRows * 16), kTcRows * 16, 128, false);
                        boff = (uint32_t)(2 * ks * NP * 16);
                    }
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        const uint64_t bd =
                            SW ? umma_smem_desc(bbase + (uint32_t)(part * part_bytes) + boff, 16,
                                                1024, true)
                               : umma_smem_desc(bbase + (uint32_t)(part * part_bytes) + boff,
                                                (uint32_t)NP * 16, 128, false);
                        umma_bf16(dacc, ad, bd, idesc, acc);
                        acc = 1;
                    }
                }
                umma_commit(bar(T_FULL + s));
                umma_commit(bar(A_EMPTY + s));
            }
        }
        __syncwarp();   // the warp reaches the final CTA barrier together
    } else {
        // ---- epilogue warps: one row per thread, a quarter of the heads per warp
        const int quad = warp & 3, part = warp >> 2;   // TMEM lane group, column quarter
        const int rtid = quad * 32 + lane;              // row of the tile this thread reads
        // D 2^-21 + 2^-16 + D 2^-24, with a margin for the rounding of the test
        const float ceps = 1.01f * ((float)D * 4.76837158203125e-07f + 1.52587890625e-05f +
                                    (float)D * 5.9604644775390625e-08f);
        TieJob *myq = tieq + warp * kTieQ;

        // the contract's fp32 fma chains of the candidates, first maximum
        auto resolve = [&](int64_t row, int h, unsigned cand) {
            const uint4 *urow = reinterpret_cast<const uint4 *>(p.u + row * D);
            float bv = 0.f;
            int best = -1;
            while (cand) {
                const int kk = __ffs(cand) - 1;
                cand &= cand - 1;
                const float *wr = p.W + ((int64_t)h * KT + kk) * D;
                float acc = 0.f;
                for (int q = 0; q < nkc; ++q) {
                    const uint4 v = __ldg(urow + q);
                    const __nv_bfloat162 *b2v = reinterpret_cast<const __nv_bfloat162 *>(&v);
                    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(wr + q * 8));
                    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(wr + q * 8 + 4));
                    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 f = __bfloat1622float2(b2v[i]);
                        acc = __fmaf_rn(wv[2 * i], f.x, acc);
                        acc = __fmaf_rn(wv[2 * i + 1], f.y, acc);
                    }
                }
                if (best < 0 || acc > bv) {
                    bv = acc;
                    best = kk;
                }
            }
            const int64_t bb = row / p.L, t = row - bb * p.L;
            p.k_out[(bb * H + h) * p.L + t] = ok ? best : -1;
        };
        // warp-collective: resolve the queued near ties, one per lane
        auto flush_ties = [&]() {
            __syncwarp();
            const int cnt = tiecnt[warp];
            for (int e = lane; e < cnt; e += 32) resolve(myq[e].row, myq[e].h, myq[e].cand);
            __syncwarp();
            if (lane == 0) tiecnt[warp] = 0;
            __syncwarp();
        };

        int j = 0;
        for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++j) {
            const int s = j & 1;
            const uint32_t ph = (uint32_t)((j >> 1) & 1);
            const int64_t row = (int64_t)tile * kTcRows + rtid;
            // partial ||u_row||^2 (this warp's quarter of the row) from the staged tile
            ok = mbar_wait_bounded(bar(A_FULL + s), ph) && ok;
            {
                const unsigned char *abase = As + (size_t)s * abytes;
                float s0 = 0.f, s1 = 0.f;
                if constexpr (SW) {
                    // this quarter of the row's (atom, 16-byte chunk) pieces; logical
                    // chunk c of row r sits at c ^ (r & 7), so the lanes of a warp
                    // hit all eight positions (no bank conflicts)
                    const int npc = (D / 64) * 8, q0 = part * (npc / 4), q1 = q0 + npc / 4;
                    for (int q = q0; q < q1; ++q) {
                        const int a = q >> 3, c = q & 7;
                        const uint4 v = *reinterpret_cast<const uint4 *>(
                            abase + a * (kTcRows * 128) + rtid * 128 + ((c ^ (rtid & 7)) << 4));
                        const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = __bfloat1622float2(b2[i]);
                            s0 = fmaf(f.x, f.x, s0);
                            s1 = fmaf(f.y, f.y, s1);
                        }
                    }
                } else {
                    const unsigned char *arow = abase + rtid * 16;
                    const int q0 = nkc * part / 4, q1 = nkc * (part + 1) / 4;
                    for (int q = q0; q < q1; ++q) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(arow + q * (kTcRows * 16));
                        const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = __bfloat1622float2(b2[i]);
                            s0 = fmaf(f.x, f.x, s0);
                            s1 = fmaf(f.y, f.y, s1);
                        }
                    }
                }
                npart[(s * 4 + part) * kTcRows + rtid] = s0 + s1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(A_EMPTY + s));
            // both halves of every row are in before any warp reads them
            asm volatile("bar.sync 1, %0;" ::"r"(kTcEpiWarps * 32) : "memory");
            // ||u_row||_2 (rounded up): round-to-nearest sums of at most 256
            // positive terms err by less than 2^-16 relative, which the factor
            // 1 + 2^-10 covers
            const float usq = (npart[(s * 4) * kTcRows + rtid] + npart[(s * 4 + 1) * kTcRows + rtid]) + (npart[(s * 4 + 2) * kTcRows + rtid] + npart[(s * 4 + 3) * kTcRows + rtid]);
            const float unorm = __fmul_ru(__fsqrt_ru(usq), 1.0009765625f);

            ok = mbar_wait_bounded(bar(T_FULL + s), ph) && ok;
            tc_fence_after();
            const bool live = row < p.rows;
            const int64_t bb = row / p.L, t = row - bb * p.L;
            auto decide = [&](const float *lg, int h) {
                float b1 = lg[0];
#pragma unroll
                for (int kk = 1; kk < KT; ++kk) b1 = fmaxf(b1, lg[kk]);
                const float S = __fmul_ru(unorm, Wn[h]);
                const float thr = b1 - 2.0f * __fmul_ru(S, ceps);
                if (p.logits_out) {
#pragma unroll
                    for (int kk = 0; kk < KT; ++kk) p.logits_out[row * (H * KT) + h * KT + kk] = lg[kk];
                    p.scale_out[row * H + h] = S;
                }
                unsigned cand = 0;
#pragma unroll
                for (int kk = 0; kk < KT; ++kk) cand |= (lg[kk] >= thr ? 1u : 0u) << kk;
                if (__popc(cand) == 1) {
                    p.k_out[(bb * H + h) * p.L + t] = ok ? __ffs(cand) - 1 : -1;
                } else {
                    // near tie (or no finite logit): exact fma chains later
                    const int slot = atomicAdd(tiecnt + warp, 1);
                    if (cand == 0) cand = (KT == 32) ? 0xffffffffu : ((1u << KT) - 1u);
                    if (slot < kTieQ) {
                        myq[slot].row = row;
                        myq[slot].h = h;
                        myq[slot].cand = cand;
                    } else {
                        resolve(row, h, cand);   // unreachable while flushes keep 32 slots free
                    }
                }
            };
            const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)s * tcols;
            if constexpr (KT <= 16) {
                // 16 columns per load hold 16 / KT whole heads; the four warps
                // of a lane group take every fourth load
                for (int c = part; c < NP / 16; c += 4) {
                    float v[16];
                    tmem_ld16(tlane + (uint32_t)(c * 16), v);
#pragma unroll
                    for (int jh = 0; jh < 16 / KT; ++jh) {
                        const int h = c * (16 / KT) + jh;
                        if (live && h < H) decide(v + jh * KT, h);
                        __syncwarp();
                        if (tiecnt[warp] > kTieQ - 32) flush_ties();
                    }
                }
            } else {
                for (int h = part; h < H; h += 4) {
                    float v[32];
                    tmem_ld16(tlane + (uint32_t)(h * 32), *reinterpret_cast<float(*)[16]>(v));
                    tmem_ld16(tlane + (uint32_t)(h * 32 + 16), *reinterpret_cast<float(*)[16]>(v + 16));
                    if (live) decide(v, h);
                    __syncwarp();
                    if (tiecnt[warp] > kTieQ - 32) flush_ties();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(T_EMPTY + s));
        }
        flush_ties();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(2u * tcols)
                     : "memory");
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            ptr = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

bool select_tc_supported(const pdssm_dims &dm, pdssm_dtype ut, const void *u, const float *W) {
    if (ut != PDSSM_BF16) return false;
    if (((uintptr_t)W % 16) != 0) return false;   // float4 reads of W rows
    const int64_t HK = dm.H * dm.K;
    const int NP = (int)((HK + 15) / 16 * 16);
    if (NP > 256 || dm.D_in % 16 != 0 || dm.D_in > 256) return false;
    if (dm.K != 1 && dm.K != 2 && dm.K != 4 && dm.K != 8 && dm.K != 16 && dm.K != 32) return false;
    if (((uintptr_t)u % 16) != 0) return false;
    if (tc_smem_bytes((int)dm.D_in, NP, (int)dm.H) > 220 * 1024) return false;
    return tensor_map_encoder() != nullptr;
}

cudaError_t launch_select_tc(const pdssm_dims &dm, const void *u, const float *W, int32_t *k_out,
                             float *logits_out, float *scale_out, cudaStream_t st) {
    const int64_t rows = dm.B * dm.L;
    const int D = (int)dm.D_in;
    const int NP = (int)((dm.H * dm.K + 15) / 16 * 16);
    // 128-byte swizzle when D is a multiple of 64 (boxes of 64 x 128), else
    // no swizzle (boxes of 8 x 128)
    const bool sw = D % 64 == 0;
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {sw ? 64u : 8u, kTcRows};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = tensor_map_encoder()(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(u),
                                      gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                      sw ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    TcSelectParams p;
    p.W = W;
    p.u = reinterpret_cast<const __nv_bfloat16 *>(u);
    p.k_out = k_out;
    p.logits_out = logits_out;
    p.scale_out = scale_out;
    p.rows = rows;
    p.L = dm.L;
    p.D = D;
    p.H = (int)dm.H;
    p.K = (int)dm.K;
    p.NP = NP;
    p.ntiles = (int)((rows + kTcRows - 1) / kTcRows);
    p.tcols = 32;
    while (p.tcols < (uint32_t)NP) p.tcols *= 2;
    const size_t smem = tc_smem_bytes(D, NP, p.H);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = p.ntiles < sms ? p.ntiles : sms;
    auto launch = [&](auto kern) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st, map, p);
    };
    if (sw) {
        switch (p.K) {
            case 1: return launch(k_select_tc<1, true>);
            case 2: return launch(k_select_tc<2, true>);
            case 4: return launch(k_select_tc<4, true>);
            case 8: return launch(k_select_tc<8, true>);
            case 16: return launch(k_select_tc<16, true>);
            default: return launch(k_select_tc<32, true>);
        }
    }
    switch (p.K) {
        case 1: return launch(k_select_tc<1, false>);
        case 2: return launch(k_select_tc<2, false>);
        case 4: return launch(k_select_tc<4, false>);
        case 8: return launch(k_select_tc<8, false>);
        case 16: return launch(k_select_tc<16, false>);
        default: return launch(k_select_tc<32, false>);
    }
}

}  // namespace pdssm
