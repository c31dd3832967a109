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
// Operand layouts in shared memory (K-major, no swizzle, 16-byte core rows):
//   A: [D/8 k-chunks][128 rows][8 bf16]     (TMA boxes of 8 x 128)
//   B: [2 parts][D/8 k-chunks][NP rows][8 bf16], NP = H*K rounded up to 16
// so a k-step of 16 covers two chunks (leading byte offset = one chunk slab)
// and rows advance by 16 bytes (stride byte offset = 128 bytes per 8 rows).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace pdssm {

constexpr int kTcRows = 128;
constexpr int kTcThreads = 256;   // two warps per group of 32 TMEM lanes

__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    // base offset 0, lbo mode 0, layout type 0 (no swizzle)
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

// Dynamic shared memory: [B parts][A x 2][row-norm partials 2 x 2 x 128]
// [tie queues 8 x kTieQ][tie counts 8][Wn H floats][barriers][tmem slot]
__host__ __device__ inline size_t tc_b_bytes(int D, int NP) { return (size_t)2 * D * NP * 2; }
__host__ __device__ inline size_t tc_a_bytes(int D) { return (size_t)kTcRows * D * 2; }
constexpr size_t kTcNormBytes = (size_t)2 * 2 * kTcRows * 4;
constexpr size_t kTcTieBytes = (size_t)(kTcThreads / 32) * kTieQ * sizeof(TieJob) + 64;
__host__ __device__ inline size_t tc_smem_bytes(int D, int NP, int H) {
    return 1024 + tc_b_bytes(D, NP) + 2 * tc_a_bytes(D) + kTcNormBytes + kTcTieBytes +
           ((size_t)H * 4 + 15) / 16 * 16 + 64;
}

template <int KT>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_select_tc(const __grid_constant__ CUtensorMap umap, const TcSelectParams p) {
    extern __shared__ __align__(1024) unsigned char sm_raw[];
    // 1024-byte alignment of the operand region
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;   // TMEM lane group, column half
    const int rtid = quad * 32 + lane;              // row of the tile this thread reads
    const int D = p.D, NP = p.NP, H = p.H, K = KT;
    const int nkc = D / 8;
    unsigned char *Bs = sm;                               // [2][nkc][NP][8] bf16
    unsigned char *As = Bs + tc_b_bytes(D, NP);           // [2][nkc][128][8] bf16
    float *npart = reinterpret_cast<float *>(As + 2 * tc_a_bytes(D));   // [2 tiles][2 halves][128]
    TieJob *tieq = reinterpret_cast<TieJob *>(reinterpret_cast<unsigned char *>(npart) + kTcNormBytes);
    int *tiecnt = reinterpret_cast<int *>(tieq + (kTcThreads / 32) * kTieQ);
    float *Wn = reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(npart) + kTcNormBytes +
                                          kTcTieBytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<unsigned char *>(Wn) +
                                                  ((size_t)H * 4 + 15) / 16 * 16);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);
    const uint32_t barA0 = smem_u32(&bars[0]), barA1 = smem_u32(&bars[1]);
    const uint32_t barM0 = smem_u32(&bars[2]), barM1 = smem_u32(&bars[3]);

    const uint32_t abytes = (uint32_t)tc_a_bytes(D);
    auto issue_a = [&](int tile, int buf) {
        const uint32_t bar = buf ? barA1 : barA0;
        mbar_expect_tx(bar, abytes);
        const uint32_t dst = smem_u32(As + (size_t)buf * abytes);
        for (int q = 0; q < nkc; ++q)
            tma_load_2d(dst + q * (kTcRows * 16), &umap, q * 8, tile * kTcRows, bar);
    };
    // barriers first, so the first tile's copy overlaps the weight split
    if (tid == 0) {
        mbar_init(barA0, 1);
        mbar_init(barA1, 1);
        mbar_init(barM0, 1);
        mbar_init(barM1, 1);
        fence_mbar_init();
        if ((int)blockIdx.x < p.ntiles) issue_a(blockIdx.x, 0);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(2u * p.tcols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int h = tid; h < H; h += kTcThreads) Wn[h] = 0.f;
    if (tid < kTcThreads / 32) tiecnt[tid] = 0;
    __syncthreads();

    // ---- weights: split into hi/lo bf16 parts in the K-major slab layout.
    // One warp per row n of W (rows past H*K are zero), four consecutive d
    // per lane, eight rows per pass so their loads are in flight together.
    // The squared row norm (rounded up) goes to the head's maximum.
    const int HK = H * K;
    constexpr int kRowsPerPass = 8;
    constexpr int kWarps = kTcThreads / 32;
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
                const size_t off = ((size_t)(d0 >> 3) * NP + n) * 16 + (d0 & 7) * 2;
                *reinterpret_cast<uint2 *>(Bs + off) = *reinterpret_cast<const uint2 *>(hi);
                *reinterpret_cast<uint2 *>(Bs + (size_t)nkc * NP * 16 + off) =
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

    // ---- tile loop, software-pipelined over two TMEM accumulators: the
    // product of tile j runs on the tensor cores while the threads decide
    // tile j - 1.  A buffer a is refilled (tile j + 1) once the product that
    // read it (tile j - 1) has completed.
    const uint32_t idesc = umma_idesc_bf16(NP);
    const uint32_t tcols = p.tcols;   // columns of one accumulator
    // D 2^-21 + 2^-16 + D 2^-24, with a margin for the rounding of the test
    const float ceps = 1.01f * ((float)D * 4.76837158203125e-07f + 1.52587890625e-05f +
                                (float)D * 5.9604644775390625e-08f);
    bool ok = true;
    int64_t row_prev = -1;
    TieJob *myq = tieq + warp * kTieQ;

    // The contract's fp32 fma chains of the candidates of one (row, head),
    // first maximum.
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

    // decide the rows of a finished tile: one row per thread, half of the
    // heads per warp
    auto epilogue = [&](int buf, int64_t row) {
        const bool live = row < p.rows;
        const int64_t bb = row / p.L, t = row - bb * p.L;
        // ||u_row||_2 (rounded up) from the halves' partial sums; the sums are
        // round-to-nearest over at most 256 positive terms, so the relative
        // error is below 2^-16 and the factor 1 + 2^-10 keeps it a bound
        const float usq = npart[(buf * 2 + 0) * kTcRows + rtid] + npart[(buf * 2 + 1) * kTcRows + rtid];
        const float unorm = __fmul_ru(__fsqrt_ru(usq), 1.0009765625f);
        auto decide = [&](const float *lg, int h) {
            float b1 = lg[0];
#pragma unroll
            for (int kk = 1; kk < KT; ++kk) b1 = fmaxf(b1, lg[kk]);
            const float thr = b1 - 2.0f * __fmul_ru(__fmul_ru(unorm, Wn[h]), ceps);
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
        const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * tcols;
        if constexpr (KT <= 16) {
            // 16 columns per load hold 16 / KT whole heads; the two warps of a
            // lane group take alternate loads
            for (int c = half; c < NP / 16; c += 2) {
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
            for (int h = half; h < H; h += 2) {
                float v[32];
                tmem_ld16(tlane + (uint32_t)(h * 32), *reinterpret_cast<float(*)[16]>(v));
                tmem_ld16(tlane + (uint32_t)(h * 32 + 16), *reinterpret_cast<float(*)[16]>(v + 16));
                if (live) decide(v, h);
                __syncwarp();
                if (tiecnt[warp] > kTieQ - 32) flush_ties();
            }
        }
    };

    int j = 0;
    for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++j) {
        const int buf = j & 1;
        const uint32_t parity = (uint32_t)((j >> 1) & 1);
        ok = mbar_wait_bounded(buf ? barA1 : barA0, parity) && ok;
        tc_fence_after();
        if (tid == 0) {
            const uint32_t abase = smem_u32(As + (size_t)buf * abytes);
            const uint32_t bbase = smem_u32(Bs);
            int acc = 0;
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t ad = umma_smem_desc(abase + 2 * ks * (kTcRows * 16),
                                                   kTcRows * 16, 128);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint64_t bd = umma_smem_desc(
                        bbase + (uint32_t)(((size_t)part * nkc + 2 * ks) * NP * 16),
                        (uint32_t)NP * 16, 128);
                    umma_bf16(tmem + (uint32_t)buf * tcols, ad, bd, idesc, acc);
                    acc = 1;
                }
            }
            umma_commit(buf ? barM1 : barM0);
        }
        // partial ||u_row||^2 of this tile (this warp's half of the row),
        // read while the product runs
        const int64_t row = (int64_t)tile * kTcRows + rtid;
        {
            const unsigned char *arow = As + (size_t)buf * abytes + rtid * 16;
            float s0 = 0.f, s1 = 0.f;
            const int q0 = half * (nkc / 2), q1 = q0 + nkc / 2;
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
            npart[(buf * 2 + half) * kTcRows + rtid] = s0 + s1;
        }
        if (j > 0) {
            // the previous tile: its product is done, so its A buffer can take
            // the tile after this one
            const int pb = buf ^ 1;
            ok = mbar_wait_bounded(pb ? barM1 : barM0, (uint32_t)(((j - 1) >> 1) & 1)) && ok;
            tc_fence_after();
            const int next = tile + gridDim.x;
            if (tid == 0 && next < p.ntiles) issue_a(next, pb);
            epilogue(pb, row_prev);
        } else {
            const int next = tile + gridDim.x;
            if (tid == 0 && next < p.ntiles) issue_a(next, buf ^ 1);
        }
        row_prev = row;
        tc_fence_before();
        __syncthreads();
    }
    if (j > 0) {
        const int pb = (j - 1) & 1;
        ok = mbar_wait_bounded(pb ? barM1 : barM0, (uint32_t)(((j - 1) >> 1) & 1)) && ok;
        tc_fence_after();
        epilogue(pb, row_prev);
    }
    flush_ties();
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
                             cudaStream_t st) {
    const int64_t rows = dm.B * dm.L;
    const int D = (int)dm.D_in;
    const int NP = (int)((dm.H * dm.K + 15) / 16 * 16);
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {8, kTcRows};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = tensor_map_encoder()(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(u),
                                      gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    TcSelectParams p;
    p.W = W;
    p.u = reinterpret_cast<const __nv_bfloat16 *>(u);
    p.k_out = k_out;
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
        kern<<<grid, kTcThreads, smem, st>>>(map, p);
        return cudaGetLastError();
    };
    switch (p.K) {
        case 1: return launch(k_select_tc<1>);
        case 2: return launch(k_select_tc<2>);
        case 4: return launch(k_select_tc<4>);
        case 8: return launch(k_select_tc<8>);
        case 16: return launch(k_select_tc<16>);
        default: return launch(k_select_tc<32>);
    }
}

}  // namespace pdssm
