// Shared device helpers and launch plumbing for the PD-SSM kernels (sm_100a).
//
// Work decomposition used by every chunk kernel: one warp owns one
// (batch, head, chunk) unit; lane l owns state elements e = l*NPL + r,
// r < NPL, NPL = ceil(N / 32) in {1, 2}.  Chunk data (rows of d, b, c) are
// contiguous in HBM, so each warp streams its chunk through shared memory in
// tiles of kTS steps with 1-D bulk copies (cp.async.bulk, the TMA engine's
// non-tensor path) completed on per-warp mbarriers: a two-stage ring (fixed
// at compile time in the fast kernels for N = 32 / 64; the general kernels
// add an L2 prefetch ahead of it).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "../../include/pdssm.h"

namespace pdssm {

constexpr int kTS = 8;         // steps per staged tile = steps per readout group
constexpr int kMaxWPC = 8;     // most warps (units) per CTA in the chunk kernels
constexpr int kMaxN = 64;
constexpr int kMaxStages = 2;
constexpr int kBwdMaxChunk = 256;   // checkpoints of one chunk kept in shared memory (general bwd C)
constexpr int kDcap = 8;            // sources per target held in the slot table
constexpr int kPrefetchTiles = 4;   // tiles prefetched into L2 ahead of the staged ones (general kernels)
constexpr int kZeroSlot = 64;       // exchange-buffer entry that always holds 0
constexpr int kPbStride = 80;       // floats per exchange buffer (64 + zero slot, padded)
constexpr unsigned kFull = 0xffffffffu;

// status word bits (first int of the workspace)
enum : int { kStBadIndex = 1, kStTimeout = 2 };

// ---------------------------------------------------------------------------
// workspace layout (all offsets 256-byte aligned)
// ---------------------------------------------------------------------------
struct WsLayout {
    size_t status, dict, tab, fan, seg, segw, look, Pi, Dl, v, Hc, wc, lam, total;
    int64_t C, Hd;
};

// Look-back region of the single-pass forward: a 64-bit chunk ticket counter
// (first 8 bytes of a 256-byte header), then one flag word per chunk.
constexpr size_t kLookHeader = 256;

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

inline WsLayout ws_layout(const pdssm_dims &dm, int64_t pi_hs, int64_t chunk,
                          bool for_bwd) {
    WsLayout w{};
    w.C = dm.L > 0 ? (dm.L + chunk - 1) / chunk : 0;
    w.Hd = pi_hs ? dm.H : 1;
    const size_t units = (size_t)(dm.B * dm.H * w.C);
    const size_t vecs = units * (size_t)dm.N * 4;
    size_t o = 0;
    w.status = o; o += 256;
    w.dict = o;   o = align256(o + (size_t)(w.Hd * dm.K * dm.N) * 4);
    w.tab = o;    o = align256(o + (size_t)(w.Hd * dm.K * kDcap * 64));
    w.fan = o;    o = align256(o + (size_t)(w.Hd * dm.K) * 4);
    w.seg = o;    o = align256(o + (size_t)(w.Hd * dm.K) * 32 * 8);
    w.segw = o;   o = align256(o + (size_t)(w.Hd * dm.K) * 32 * 8);
    w.look = o;   o = align256(o + kLookHeader + units * 4);
    w.Pi = o;     o = align256(o + vecs);
    w.Dl = o;     o = align256(o + vecs);
    w.v = o;      o = align256(o + vecs);
    w.Hc = o;     o = align256(o + vecs);
    if (for_bwd) {
        w.wc = o;  o = align256(o + vecs);
        w.lam = o; o = align256(o + vecs);
    }
    w.total = o;
    return w;
}

// ---------------------------------------------------------------------------
// parameters of the chunk kernels
// ---------------------------------------------------------------------------
struct ChunkParams {
    int64_t B, H, L, N, K, C, chunk, units;
    int64_t dict_hs;          // head stride of the sanitised dictionary (0 or K*N)
    const int32_t *dict;      // sanitised dictionary [Hd][K][N]
    const uint8_t *tab;       // slot tables [Hd][K][kDcap][64]: s-th source of each target
    const int32_t *fan;       // largest fan-in of each map [Hd][K]
    const uint2 *seg;         // segment tables [Hd][K][32 lanes] (N = 32 or 64)
    const uint2 *segw;        // window tables [Hd][K][32 lanes] (N = 64)
    const int *dict_stats;    // over all maps: [0] largest lane distance inside a
                              // segment, [1] largest fan-in (1: all permutations),
                              // [2] largest back-span of the window tables (N = 64)
    int dict_content;         // parts of the dictionary staged in shared memory
    const int32_t *k;
    const void *d, *b, *c;
    const float *h0;
    float *y;
    int32_t *Pi;
    float *Dl, *v, *Hc, *wc, *lam;
    const float *g_y, *g_hlast;
    float *g_b, *g_d, *g_c, *g_h0;
    float *h_last;
    int *status;
    int *look;                // single-pass forward: per-chunk flags (0, kFlagAgg, kFlagIncl)
    unsigned long long *ticket;   // single-pass forward: next chunk ticket
    uint64_t wait_ns;         // cap of every bounded wait, in ns of the global timer
    // selection inside the single-pass forward (k never leaves the CTA)
    const void *u;            // bf16 [B][L][D_in]
    const float *W_sel;       // [H][K][D_in]
    int D_in;
    int32_t *k_out;           // optional copy of the selection [B][H][L]
    int ns;                   // pipeline stages
    int wpc;                  // warps (units) per CTA
    int bulk;                 // 1: bulk-copy staging; 0: cooperative copies
    int smem_per_warp;
};

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void flag_status(int *status, int bit) {
    atomicOr(status, bit);
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier.  Plain
// per-CTA copy of this GPU's own memory, delivered to this CTA only.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], "
        "%2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Bulk prefetch of global memory into L2 (no shared memory involved).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Cap of every bounded wait (global-timer ns) unless a caller passes another.
constexpr uint64_t kWaitCapNs = 2000000000ull;

// Bounded wait: gives up after cap_ns of wall time or 2^26 polls.
static __device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                      uint64_t cap_ns = kWaitCapNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 26); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 1023u) == 1023u && global_ns() - t0 > cap_ns) break;
    }
    return false;
}

// Flag words shared between CTAs of one grid (single-pass forward): the
// writer stores its data, fences, and publishes the flag with a release
// store; the reader polls with acquire loads and reads the data through L2.
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int *p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// explicit 32-bit shared-memory accesses for the hot loops
// ---------------------------------------------------------------------------
__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float2 lds_f32x2(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}
// Shared loads at a compile-time byte offset from a register address.
template <int OFF>
__device__ __forceinline__ unsigned lds_u16_at(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1+%2];" : "=h"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ float lds_f32_at(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
    return v;
}
// element of a staged row at byte address a + OFF, as float
template <typename T, int OFF>
__device__ __forceinline__ float lds_elem_at(uint32_t a) {
    if constexpr (sizeof(T) == 4)
        return lds_f32_at<OFF>(a);
    else
        return __uint_as_float(lds_u16_at<OFF>(a) << 16);
}
// next column position (a byte offset idx * sizeof(T)) through a map staged
// with entries of sizeof(T) bytes
template <typename T>
__device__ __forceinline__ int lds_next_pos(uint32_t a) {
    if constexpr (sizeof(T) == 4) {
        int v;
        asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(a));
        return v;
    } else {
        return (int)lds_u16_at<0>(a);
    }
}

__device__ __forceinline__ uint2 lds_u32x2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ int lds_s32(uint32_t a) {
    int v;
    asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ int2 lds_s32x2(uint32_t a) {
    int2 v;
    asm volatile("ld.shared.v2.s32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ unsigned lds_u8(uint32_t a) {
    unsigned v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ unsigned lds_u16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ unsigned lds_u32(uint32_t a) {
    unsigned v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void sts_f32x2(uint32_t a, float x, float y) {
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(x), "f"(y) : "memory");
}
__device__ __forceinline__ void warp_barrier() {
    asm volatile("bar.warp.sync -1;" ::: "memory");
}
// One element of type T at a shared address, as float.
template <typename T>
__device__ __forceinline__ float lds_elem(uint32_t a);
template <>
__device__ __forceinline__ float lds_elem<float>(uint32_t a) { return lds_f32(a); }
template <>
__device__ __forceinline__ float lds_elem<__nv_bfloat16>(uint32_t a) {
    return __uint_as_float(lds_u16(a) << 16);
}
// Two consecutive elements of type T at a shared address (8- or 4-aligned).
template <typename T>
__device__ __forceinline__ float2 lds_pair(uint32_t a);
template <>
__device__ __forceinline__ float2 lds_pair<float>(uint32_t a) { return lds_f32x2(a); }
template <>
__device__ __forceinline__ float2 lds_pair<__nv_bfloat16>(uint32_t a) {
    const unsigned w = lds_u32(a);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// The same loads and stores at a compile-time byte offset from a register
// address (for fully unrolled tiles).
template <int OFF>
__device__ __forceinline__ unsigned lds_u32_at(uint32_t a) {
    unsigned v;
    asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ float2 lds_f32x2_at(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2+%3];" : "=f"(v.x), "=f"(v.y) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ void sts_f32_at(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0+%1], %2;" ::"r"(a), "n"(OFF), "f"(v) : "memory");
}
template <typename T, int OFF>
__device__ __forceinline__ float2 lds_pair_at(uint32_t a) {
    if constexpr (sizeof(T) == 4) {
        return lds_f32x2_at<OFF>(a);
    } else {
        const unsigned w = lds_u32_at<OFF>(a);
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
}

// Calls f(std::integral_constant<int, Q>) for Q = 0 .. sizeof...(Qs) - 1 in
// order (a loop unrolled at compile time).
template <typename F, int... Qs>
__device__ __forceinline__ void for_each_q(F &&f, std::integer_sequence<int, Qs...>) {
    (f(std::integral_constant<int, Qs>{}), ...);
}

// Load the NPL elements a lane owns from one staged row (0 beyond N).
template <typename T, int NPL, bool EVEN>
__device__ __forceinline__ void load_row(const T *row, int lane, int N, float (&v)[NPL]) {
    if constexpr (NPL == 1) {
        v[0] = lane < N ? to_f<T>(row[lane]) : 0.f;
    } else {
        const int e0 = 2 * lane;
        if constexpr (EVEN) {
            if (e0 < N) {
                if constexpr (std::is_same<T, float>::value) {
                    const float2 q = *reinterpret_cast<const float2 *>(row + e0);
                    v[0] = q.x;
                    v[1] = q.y;
                } else {
                    const __nv_bfloat162 q = *reinterpret_cast<const __nv_bfloat162 *>(row + e0);
                    v[0] = __low2float(q);
                    v[1] = __high2float(q);
                }
            } else {
                v[0] = 0.f;
                v[1] = 0.f;
            }
        } else {
            v[0] = e0 < N ? to_f<T>(row[e0]) : 0.f;
            v[1] = e0 + 1 < N ? to_f<T>(row[e0 + 1]) : 0.f;
        }
    }
}

// Selection index of one step, clamped into [0, K) (flagged when it was not).
__device__ __forceinline__ int clamp_k(int kv, int K, int *status) {
    if (kv < 0 || kv >= K) {
        flag_status(status, kStBadIndex);
        kv = kv < 0 ? 0 : K - 1;
    }
    return kv;
}
__device__ __forceinline__ int load_k(const int32_t *kp, int64_t idx, bool valid, int K,
                                      int *status) {
    return clamp_k(valid ? __ldg(kp + idx) : 0, K, status);
}
// Raw load of the next tile's indices; clamp_k them only when they are used,
// so the load's latency is hidden behind the current tile.
__device__ __forceinline__ int load_k_raw(const int32_t *kp, int64_t idx, bool valid) {
    return valid ? __ldg(kp + idx) : 0;
}

// ---------------------------------------------------------------------------
// dictionary in shared memory and the PD step as a shared-memory scatter
// ---------------------------------------------------------------------------

// Loads the NPL elements a lane owns from one staged row.  FULL means the
// state fills the warp (N == 32 * NPL): no guards, vector loads.
template <typename T, int NPL, bool FULL>
__device__ __forceinline__ void ld_own(const T *row, int lane, int N, float (&v)[NPL]) {
    if constexpr (FULL) {
        if constexpr (NPL == 1) {
            v[0] = to_f<T>(row[lane]);
        } else if constexpr (std::is_same<T, float>::value) {
            const float2 q = *reinterpret_cast<const float2 *>(row + 2 * lane);
            v[0] = q.x;
            v[1] = q.y;
        } else {
            const __nv_bfloat162 q = *reinterpret_cast<const __nv_bfloat162 *>(row + 2 * lane);
            v[0] = __low2float(q);
            v[1] = __high2float(q);
        }
    } else {
#pragma unroll
        for (int r = 0; r < NPL; ++r) {
            const int e = lane * NPL + r;
            v[r] = e < N ? to_f<T>(row[e]) : 0.f;
        }
    }
}

// One PD step h <- P_k diag(d) h + b on the lane-owned state, as a gather:
// every lane stores d[j] h[j] of the sources it owns into `pb` (this step's
// buffer of an alternating pair, entry kZeroSlot permanently 0), then sums,
// for each element it owns, the sources listed by the map's slot table in
// ascending j (padding entries point at the zero slot).  One warp barrier per
// step; no atomics, so the result is deterministic.  `tabl` is the map's
// table advanced to this lane's first element; Dk the map's largest fan-in
// (maps above kDcap scan all N sources instead).
template <int NPL, bool FULL>
__device__ __forceinline__ void pd_gather_step(float (&h)[NPL], const float (&dv)[NPL],
                                               const float (&bv)[NPL], float *pb,
                                               const uint8_t *tabl, int Dk, const int *pk,
                                               int lane, int N) {
    if constexpr (NPL == 2) {
        if (FULL || 2 * lane + 1 < N) {
            *reinterpret_cast<float2 *>(pb + 2 * lane) = make_float2(dv[0] * h[0], dv[1] * h[1]);
        } else if (2 * lane < N) {
            pb[2 * lane] = dv[0] * h[0];
        }
    } else {
        if (FULL || lane < N) pb[lane] = dv[0] * h[0];
    }
    __syncwarp();
    float acc[NPL];
    if (Dk <= kDcap) {
        if constexpr (NPL == 2) {
            unsigned w = *reinterpret_cast<const uint16_t *>(tabl);
            acc[0] = pb[w & 0xffu];
            acc[1] = pb[w >> 8];
            for (int sl = 1; sl < Dk; ++sl) {
                w = *reinterpret_cast<const uint16_t *>(tabl + sl * 64);
                acc[0] += pb[w & 0xffu];
                acc[1] += pb[w >> 8];
            }
        } else {
            acc[0] = pb[tabl[0]];
            for (int sl = 1; sl < Dk; ++sl) acc[0] += pb[tabl[sl * 64]];
        }
    } else {
#pragma unroll
        for (int r = 0; r < NPL; ++r) acc[r] = 0.f;
        for (int j = 0; j < N; ++j) {
            const int t = pk[j];
            const float v = pb[j];
#pragma unroll
            for (int r = 0; r < NPL; ++r)
                if (t == lane * NPL + r) acc[r] += v;
        }
    }
#pragma unroll
    for (int r = 0; r < NPL; ++r) h[r] = (FULL || lane * NPL + r < N) ? acc[r] + bv[r] : 0.f;
}

// Sum over the warp of per-step partials staged in ybuf[q][33] (kTS = 8
// rows): lane l adds 8 entries of row l / 4, two shuffles combine the four
// quarters, and lane 4 q ends up with the total of row q.  Conflict-free.
// Caller synchronises before; every lane must call it.
__device__ __forceinline__ float ybuf_quad_sum(const float *ybuf, int lane) {
    static_assert(kTS == 8, "quarter-row reduction assumes 8 rows");
    const float *src = ybuf + (lane >> 2) * 33 + (lane & 3) * 8;
    float s = src[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) s += src[i];
    s += __shfl_xor_sync(kFull, s, 1);
    s += __shfl_xor_sync(kFull, s, 2);
    return s;
}

// Sum over the warp of per-step partials staged in ybuf[q][33] (rows
// q < n): lane q < n returns the total of row q.  Caller synchronises.
__device__ __forceinline__ float ybuf_row_sum(const float *ybuf, int lane, int n) {
    float s = 0.f;
    if (lane < n) {
        const float *row = ybuf + lane * 33;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) s += row[j];
    }
    return s;
}

// Both exchange buffers of a warp: zero, including the zero slots.
__device__ __forceinline__ void clear_pb(float *pb, int lane) {
    for (int i = lane; i < 2 * kPbStride; i += 32) pb[i] = 0.f;
    __syncwarp();
}

// ---------------------------------------------------------------------------
// per-warp staging ring: NT tensors, ns stages of kTS rows each
// ---------------------------------------------------------------------------
template <int NT>
struct Ring {
    unsigned char *buf;    // stage 0, tensor 0
    uint32_t bar0;         // mbarrier of stage 0 (8 bytes each)
    int stage_bytes;       // NT * tens_bytes
    int tens_bytes;        // kTS * rowb
    int rowb;              // N * element size
    int esz;
    int ns;
    bool bulk;
    const unsigned char *src[NT];   // row 0 of this (b, h) sequence, per tensor

    __device__ unsigned char *tile(int stage, int q) const {
        return buf + stage * stage_bytes + q * tens_bytes;
    }

    // Stage rows [t0, t0 + n) of the first nt tensors into `stage`.
    __device__ void issue(int stage, int64_t t0, int n, int nt, int lane) const {
        if (bulk) {
            if (lane == 0) {
                const uint32_t bar = bar0 + 8u * stage;
                const uint32_t bytes = (uint32_t)(n * rowb);
                mbar_expect_tx(bar, bytes * (uint32_t)nt);
#pragma unroll
                for (int q = 0; q < NT; ++q)
                    if (q < nt) bulk_g2s(smem_u32(tile(stage, q)), src[q] + t0 * rowb, bytes, bar);
            }
        } else {
            const int elems = n * (rowb / esz);
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                if (q >= nt) continue;
                if (esz == 4) {
                    const float *s = reinterpret_cast<const float *>(src[q] + t0 * rowb);
                    float *dst = reinterpret_cast<float *>(tile(stage, q));
                    for (int i = lane; i < elems; i += 32) dst[i] = s[i];
                } else {
                    const unsigned short *s =
                        reinterpret_cast<const unsigned short *>(src[q] + t0 * rowb);
                    unsigned short *dst = reinterpret_cast<unsigned short *>(tile(stage, q));
                    for (int i = lane; i < elems; i += 32) dst[i] = s[i];
                }
            }
            __syncwarp();
        }
    }

    // Pull rows [t0, t0 + n) of the first nt tensors towards L2 so that the
    // later staging copy of them hits L2 instead of waiting on HBM.
    __device__ void prefetch(int64_t t0, int n, int nt, int lane) const {
        if (bulk && lane == 0 && n > 0) {
            const uint32_t bytes = (uint32_t)(n * rowb);
#pragma unroll
            for (int q = 0; q < NT; ++q)
                if (q < nt) bulk_prefetch_l2(src[q] + t0 * rowb, bytes);
        }
    }

    __device__ bool wait(int stage, uint32_t parity) const {
        if (!bulk) return true;
        return mbar_wait_bounded(bar0 + 8u * stage, parity);
    }
};

// Two-stage bulk-copy ring with compile-time geometry, for the fast-path
// kernels (N = 32 / 64, aligned rows): tile i of a chunk goes to stage i & 1
// and completes phase (i >> 1) & 1 of that stage's mbarrier.  NT tensors are
// allocated per stage; the first `nt` of them are copied.  (No L2 prefetch
// ahead of the ring: with many warps per SM in flight it measured slower.)
constexpr int kFastStages = 2;

__device__ __forceinline__ bool mbar_wait_fast(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_bounded(bar, parity);
}

template <int NT, int ROWB>
struct FastRing {
    static constexpr int TENS = kTS * ROWB;
    static constexpr int STAGEB = NT * TENS;
    uint32_t ring_s;                  // shared address of stage 0, tensor 0
    uint32_t bar0;                    // mbarrier of stage 0 (8 bytes each)
    int len;                          // rows of this chunk
    int nt;                           // tensors copied per tile
    const unsigned char *src[NT];     // row 0 of this chunk, per tensor

    __device__ uint32_t tile(int i) const { return ring_s + (uint32_t)((i & 1) * STAGEB); }

    // Copy chunk tile ti into stage m & 1: the tensors whose bits are set in
    // `mask` (bit q: tensor q).
    __device__ void issue_tile(int m, int ti, unsigned mask, int lane) const {
        if (lane == 0) {
            const int stage = m & 1;
            const uint32_t bytes = (uint32_t)(min(kTS, len - ti * kTS) * ROWB);
            const uint32_t bar = bar0 + 8u * stage;
            mbar_expect_tx(bar, bytes * (uint32_t)__popc(mask));
#pragma unroll
            for (int q = 0; q < NT; ++q)
                if ((mask >> q) & 1u)
                    bulk_g2s(ring_s + (uint32_t)(stage * STAGEB + q * TENS),
                             src[q] + (size_t)ti * TENS, bytes, bar);
        }
    }
    __device__ void issue(int i, int lane) const { issue_tile(i, i, (1u << nt) - 1u, lane); }

    __device__ bool wait(int i) const {
        return mbar_wait_fast(bar0 + 8u * (uint32_t)(i & 1), (uint32_t)((i >> 1) & 1));
    }

    // After a wait gave up on tile i: record it, then wait (bounded) for the
    // copies still in flight (tiles i and i + 1) so none lands after exit.
    __device__ void abort(int i, int ntiles, int *status, int lane) const {
        if (lane == 0) flag_status(status, kStTimeout);
        for (int j = i; j < ntiles && j < i + kFastStages; ++j) wait(j);
        __syncwarp();
    }
};

// Initialise a warp's ns mbarriers (one arrival each: the expect_tx).
__device__ __forceinline__ void ring_init_bars(uint32_t bar0, int ns, int lane) {
    if (lane == 0) {
        for (int s = 0; s < ns; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
}

// After a wait gave up: record it and wait (bounded) for the copies this warp
// still has in flight into tiles [first, last) so none lands after exit.
template <int NT>
__device__ void ring_abort(const Ring<NT> &ring, int first, int last, int *status,
                           int lane) {
    if (lane == 0) flag_status(status, kStTimeout);
    for (int i = first; i < last; ++i) ring.wait(i % ring.ns, (uint32_t)((i / ring.ns) & 1));
    __syncwarp();
}

// Dynamic shared memory of the chunk kernels:
//   [dictionary slots][warp 0][warp 1]...
//   dictionary slot = [map K x N ints][slot tables K x kDcap x 64 bytes][fan-in K ints]
//   warp = [staging ring][exchange buffers 2 x kPbStride floats]
//          [readout buffer kTS x 33 floats][extra][barriers]
constexpr int kYbufFloats = kTS * 33;
// Parts of the dictionary a kernel stages in shared memory (bit mask; 0
// means map + slot tables).
// kDictMap16: the map with 2-byte entries (for bf16 rows: entry = index * 2).
enum : int { kDictMap = 1, kDictTab = 2, kDictSeg = 4, kDictMap16 = 8 };
__host__ __device__ inline int dict_parts(int content) {
    return content ? content : (kDictMap | kDictTab);
}
__host__ __device__ inline int dict_map_bytes(int K, int N, int content = 0) {
    return (content & kDictMap16) ? (K * N * 2 + 7) / 8 * 8 : K * N * 4;
}
__host__ __device__ inline int dict_tab_bytes(int K) { return K * kDcap * 64 + K * 4; }
__host__ __device__ inline int dict_seg_bytes(int K) { return K * 32 * 8; }
__host__ __device__ inline int dict_slot_bytes(int K, int N, int content = 0) {
    const int c = dict_parts(content);
    int b = dict_map_bytes(K, N, c);
    if (c & kDictTab) b += dict_tab_bytes(K);
    if (c & kDictSeg) b = (b + 7) / 8 * 8 + dict_seg_bytes(K);
    return (b + 255) / 256 * 256;
}
__host__ __device__ inline int warp_smem_bytes(int ns, int nt, int rowb, int extra = 0) {
    return (ns * nt * kTS * rowb + 2 * kPbStride * 4 + kYbufFloats * 4 + extra + kMaxStages * 8 +
            255) / 256 * 256;
}
// The dynamic shared memory of the chunk kernels, rounded up to 256 bytes
// (launches add 256 bytes of slack), so that the per-warp regions, whose
// sizes are multiples of 256, start 256-byte aligned.
__device__ __forceinline__ unsigned char *smem_base256(unsigned char *raw) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(raw) + 255) &
                                             ~uintptr_t(255));
}

// Step variant for a launch: 0 when every map is a permutation; kStepWin
// (N = 64) when every map's window table reaches back at most two lanes;
// else the shuffle levels of the segment tables: the smallest LV in
// {1, 2, 3, 5} with 2^LV above the largest lane distance inside a segment.
constexpr int kStepWin = 8;
__device__ __forceinline__ int step_variant(const int *dict_stats, int npl) {
    if (__ldg(dict_stats + 1) <= 1) return 0;
    if (npl == 2 && __ldg(dict_stats + 2) <= 2) return kStepWin;
    const int md = __ldg(dict_stats);
    return md < 2 ? 1 : md < 4 ? 2 : md < 8 ? 3 : 5;
}

struct SmemDict {
    const int *map;        // [K][N] (2-byte entries with kDictMap16)
    const uint8_t *tab;    // [K][kDcap][64]
    const int *fan;        // [K]
    const uint2 *seg;      // [K][32]
};

__device__ __forceinline__ void copy_slot(unsigned char *dst, const ChunkParams &p, int64_t dk,
                                          int tid, int nthr, int scale) {
    const int K = (int)p.K, N = (int)p.N;
    const int c = dict_parts(p.dict_content);
    const int32_t *gm = p.dict + dk * K * N;
    if (c & kDictMap16) {
        uint16_t *m = reinterpret_cast<uint16_t *>(dst);
        for (int i = tid; i < K * N; i += nthr) m[i] = (uint16_t)(__ldg(gm + i) * scale);
    } else {
        int *m = reinterpret_cast<int *>(dst);
        for (int i = tid; i < K * N; i += nthr) m[i] = __ldg(gm + i) * scale;
    }
    int off = dict_map_bytes(K, N, c);
    if (c & kDictTab) {
        uint32_t *t = reinterpret_cast<uint32_t *>(dst + off);
        int *f = reinterpret_cast<int *>(dst + off + K * kDcap * 64);
        const uint32_t *gt = reinterpret_cast<const uint32_t *>(p.tab + dk * K * kDcap * 64);
        const int32_t *gf = p.fan + dk * K;
        for (int i = tid; i < K * kDcap * 16; i += nthr) t[i] = __ldg(gt + i);
        for (int i = tid; i < K; i += nthr) f[i] = __ldg(gf + i);
        off += dict_tab_bytes(K);
    }
    if (c & kDictSeg) {
        off = (off + 7) / 8 * 8;
        uint2 *g = reinterpret_cast<uint2 *>(dst + off);
        const bool win = N == 64 && step_variant(p.dict_stats, 2) == kStepWin;
        const uint2 *gs = (win ? p.segw : p.seg) + dk * K * 32;
        for (int i = tid; i < K * 32; i += nthr) g[i] = __ldg(gs + i);
    }
}

// View of one staged dictionary slot.
__device__ __forceinline__ SmemDict dict_view(const ChunkParams &p, const unsigned char *mine) {
    const int K = (int)p.K, N = (int)p.N;
    const int c = dict_parts(p.dict_content);
    SmemDict sd;
    sd.map = reinterpret_cast<const int *>(mine);
    int off = dict_map_bytes(K, N, c);
    sd.tab = nullptr;
    sd.fan = nullptr;
    sd.seg = nullptr;
    if (c & kDictTab) {
        sd.tab = mine + off;
        sd.fan = reinterpret_cast<const int *>(mine + off + K * kDcap * 64);
        off += dict_tab_bytes(K);
    }
    if (c & kDictSeg) sd.seg = reinterpret_cast<const uint2 *>(mine + (off + 7) / 8 * 8);
    return sd;
}

// Loads the dictionary used by this CTA's warps into shared memory and
// returns this warp's view.  Must be reached by every thread of the CTA.
// scale = 4 stores map entries as byte offsets into int32 rows.
__device__ __forceinline__ SmemDict stage_dict(const ChunkParams &p, unsigned char *smem,
                                               int warp, int lane, int scale = 1) {
    const int K = (int)p.K, N = (int)p.N;
    const int c = dict_parts(p.dict_content);
    const int slot = dict_slot_bytes(K, N, p.dict_content);
    unsigned char *mine = smem;
    if (p.dict_hs == 0) {
        copy_slot(smem, p, 0, threadIdx.x, blockDim.x, scale);
    } else {
        mine = smem + warp * slot;
        const int64_t unit = (int64_t)blockIdx.x * p.wpc + warp;
        if (unit < p.units) copy_slot(mine, p, (unit / p.C) % p.H, lane, 32, scale);
    }
    __syncthreads();
    SmemDict sd;
    sd.map = reinterpret_cast<const int *>(mine);
    int off = dict_map_bytes(K, N, c);
    sd.tab = nullptr;
    sd.fan = nullptr;
    sd.seg = nullptr;
    if (c & kDictTab) {
        sd.tab = mine + off;
        sd.fan = reinterpret_cast<const int *>(mine + off + K * kDcap * 64);
        off += dict_tab_bytes(K);
    }
    if (c & kDictSeg) sd.seg = reinterpret_cast<const uint2 *>(mine + (off + 7) / 8 * 8);
    return sd;
}

__host__ __device__ inline int dict_region_bytes(const ChunkParams &p) {
    return (p.dict_hs == 0 ? 1 : p.wpc) * dict_slot_bytes((int)p.K, (int)p.N, p.dict_content);
}

// ---------------------------------------------------------------------------
// fast-path helpers (state filling the warp: N = 32 * NPL)
// ---------------------------------------------------------------------------
template <typename T, int NPL>
__device__ __forceinline__ void lds_own(uint32_t a, float (&v)[NPL]) {
    if constexpr (NPL == 1) {
        v[0] = lds_elem<T>(a);
    } else {
        const float2 q = lds_pair<T>(a);
        v[0] = q.x;
        v[1] = q.y;
    }
}

template <typename T, int NPL, int OFF>
__device__ __forceinline__ void lds_own_at(uint32_t a, float (&v)[NPL]) {
    if constexpr (NPL == 1) {
        v[0] = lds_elem_at<T, OFF>(a);
    } else {
        const float2 q = lds_pair_at<T, OFF>(a);
        v[0] = q.x;
        v[1] = q.y;
    }
}

// The PD step through the map's segment table.  The sources of the step's
// map, sorted by target (ascending j within a target), are dealt out NPL
// per lane in order, so every target's sources form one segment of
// consecutive entries.  Each lane loads its entries' d * h, a segmented
// inclusive scan over the lanes (LV shuffle levels; 2^LV must exceed the
// largest lane distance inside a segment) sums every segment, and each
// owner fetches its targets' sums by shuffle from the lane holding the entry
// that ends the segment, then adds b.  The cost does not depend on the
// fan-in, and the sum of each target follows a fixed tree, so the step is
// deterministic.
//
// Entry word e (per map and lane):
//   e.x: byte offsets (index * 4) of source a, source b, target a, target b
//   e.y: bits 0-7 lane distance back to the start of b's segment;
//        bit 8 a and b share a target; bit 9 a continues the previous
//        lane's segment; bit 10 b ends its segment; bits 11, 12 this lane's
//        own targets (NPL e, NPL e + 1) have sources; bits 16-20 / 21 the
//        lane and entry (0: a, 1: b) ending the first own target's segment,
//        bits 22-26 / 27 the same for the second.
// With NPL = 1 a lane holds only entry b.  pb holds d * h by element; it is
// 256-byte aligned and callers alternate two such buffers on consecutive
// steps (one barrier per step).
template <int NPL, int LV>
__device__ __forceinline__ void step_seg(float (&h)[NPL], const float (&dv)[NPL],
                                         const float (&bv)[NPL], uint32_t pb, uint2 e,
                                         int lane) {
    if constexpr (NPL == 1)
        sts_f32(pb + lane * 4, dv[0] * h[0]);
    else
        sts_f32x2(pb + lane * 8, dv[0] * h[0], dv[1] * h[1]);
    warp_barrier();
    // an entry's byte offset replaces the low byte of the buffer address
    const uint32_t w0 = e.x, w1 = e.y;
    const float zb = lds_f32(__byte_perm(w0, pb, 0x7651));
    float za = 0.f, v = zb;
    bool ab_same = false;
    if constexpr (NPL == 2) {
        za = lds_f32(__byte_perm(w0, pb, 0x7650));
        ab_same = (w1 >> 8) & 1u;
        if (ab_same) v = za + zb;
    }
    const int dist = (int)(w1 & 0xffu);
#pragma unroll
    for (int o = 1; o < (1 << LV); o <<= 1) {
        const float t = __shfl_up_sync(kFull, v, o);
        if (dist >= o) v = t + v;
    }
    // v: the sum of b's segment up to b; sa: the sum of a's segment up to a
    if constexpr (NPL == 1) {
        const float x = __shfl_sync(kFull, v, (int)((w1 >> 16) & 31u));
        h[0] = ((w1 >> 11) & 1u ? x : 0.f) + bv[0];
    } else {
        const float left = __shfl_up_sync(kFull, v, 1);
        const float sa = ((w1 >> 9) & 1u) ? left + za : za;
        const int l0 = (int)((w1 >> 16) & 31u), l1 = (int)((w1 >> 22) & 31u);
        const float a0 = __shfl_sync(kFull, sa, l0), b0 = __shfl_sync(kFull, v, l0);
        const float a1 = __shfl_sync(kFull, sa, l1), b1 = __shfl_sync(kFull, v, l1);
        const float x0 = ((w1 >> 21) & 1u) ? b0 : a0;
        const float x1 = ((w1 >> 27) & 1u) ? b1 : a1;
        h[0] = ((w1 >> 11) & 1u ? x0 : 0.f) + bv[0];
        h[1] = ((w1 >> 12) & 1u ? x1 : 0.f) + bv[1];
    }
}

// The PD step when every map of the dictionary is a permutation (fan-in 1):
// a map's segment table then lists, for this lane's own targets, their only
// sources (entries NPL*lane .. NPL*lane+NPL-1 are the lane's targets).  With
// N = 32 the source's d * h comes by one shuffle; with N = 64 through the
// exchange buffer pb, which callers alternate between two 256-byte aligned
// buffers on consecutive steps (one barrier per step).
template <int NPL>
__device__ __forceinline__ void step_perm(float (&h)[NPL], const float (&dv)[NPL],
                                          const float (&bv)[NPL], uint32_t pb, uint2 e,
                                          int lane) {
    if constexpr (NPL == 1) {
        const float hd = dv[0] * h[0];
        h[0] = __shfl_sync(kFull, hd, (int)((e.x >> 10) & 31u)) + bv[0];
    } else {
        sts_f32x2(pb + lane * 8, dv[0] * h[0], dv[1] * h[1]);
        warp_barrier();
        h[0] = lds_f32(__byte_perm(e.x, pb, 0x7650)) + bv[0];
        h[1] = lds_f32(__byte_perm(e.x, pb, 0x7651)) + bv[1];
    }
}

// The PD step through the map's window table (N = 64, two entries per
// lane).  The map's targets are ordered by decreasing fan-in, each target's
// sources (ascending j) forming one segment of consecutive entries, with a
// single-source target moved in front of an even-sized segment that would
// otherwise start at an odd entry; so a segment of up to six sources
// reaches back at most two lanes from the lane holding its last entry.
// Each lane forms the partial of its last segment inside the lane ("tail"),
// and a segment that continues into the lane from the left gets the tails of
// the D <= 2 lanes it spans, fetched by two independent shuffles (no
// dependent scan levels).  The owners of the targets then fetch each
// segment's sum from the lane holding its last entry.  d * h goes to
// per-map slots of the exchange buffer chosen (a bank colouring of the
// bipartite graph of writer and reader instructions) so that both stores
// and both gathers of a step touch 32 distinct banks.
//
// Entry word e (per map and lane):
//   e.x: byte offsets (slot * 4) of source a, source b, the slot this lane
//        writes element 2 * lane to, and the slot of element 2 * lane + 1
//   e.y: bit 0 a and b share a target; bit 1 a continues the previous lane's
//        segment; bits 2-3 D, the lanes back to the start of a's segment
//        (when bit 1 is set); bits 4, 5 this lane's own targets have sources;
//        bits 16-20 / 21 the lane and entry (0: a, 1: b) ending the first own
//        target's segment, bits 22-26 / 27 the same for the second.
// The sum of each target follows a fixed order, so the step is
// deterministic.  pb is 256-byte aligned; callers alternate two buffers.
__device__ __forceinline__ void step_win(float (&h)[2], const float (&dv)[2], const float (&bv)[2],
                                         uint32_t pb, uint2 e) {
    const uint32_t w0 = e.x, w1 = e.y;
    sts_f32(__byte_perm(w0, pb, 0x7652), dv[0] * h[0]);
    sts_f32(__byte_perm(w0, pb, 0x7653), dv[1] * h[1]);
    warp_barrier();
    const float za = lds_f32(__byte_perm(w0, pb, 0x7650));
    const float zb = lds_f32(__byte_perm(w0, pb, 0x7651));
    const bool ab_same = w1 & 1u;
    const float tail = ab_same ? za + zb : zb;
    const float t1 = __shfl_up_sync(kFull, tail, 1);
    const float t2 = __shfl_up_sync(kFull, tail, 2);
    const uint32_t D = (w1 >> 2) & 3u;
    float back = D >= 1u ? t1 : 0.f;
    if (D >= 2u) back += t2;
    // sa: the sum of a's segment up to a; v: the sum of b's segment up to b
    const float sa = ((w1 >> 1) & 1u) ? za + back : za;
    const float v = ab_same ? sa + zb : zb;
    const int l0 = (int)((w1 >> 16) & 31u), l1 = (int)((w1 >> 22) & 31u);
    const float a0 = __shfl_sync(kFull, sa, l0), b0 = __shfl_sync(kFull, v, l0);
    const float a1 = __shfl_sync(kFull, sa, l1), b1 = __shfl_sync(kFull, v, l1);
    const float x0 = ((w1 >> 21) & 1u) ? b0 : a0;
    const float x1 = ((w1 >> 27) & 1u) ? b1 : a1;
    h[0] = ((w1 >> 4) & 1u ? x0 : 0.f) + bv[0];
    h[1] = ((w1 >> 5) & 1u ? x1 : 0.f) + bv[1];
}

// One PD step: LV = 0 selects the permutation step, kStepWin the window
// step (N = 64), otherwise the segment-table step with LV shuffle levels;
// each takes the exchange buffer of the step's parity (pb or ob).
template <int NPL, int LV>
__device__ __forceinline__ void pd_step(float (&h)[NPL], const float (&dv)[NPL],
                                        const float (&bv)[NPL], uint32_t pb, uint32_t ob,
                                        uint2 e, int lane, int parity) {
    if constexpr (LV == 0) {
        step_perm<NPL>(h, dv, bv, parity ? ob : pb, e, lane);
    } else if constexpr (LV == kStepWin) {
        static_assert(NPL == 2, "the window step serves N = 64");
        step_win(h, dv, bv, parity ? ob : pb, e);
    } else {
        step_seg<NPL, LV>(h, dv, bv, parity ? ob : pb, e, lane);
    }
}


// Programmatic dependent launch: a kernel launched with launch_pdl may start
// while its predecessor in the stream finishes; pdl_wait() blocks until the
// predecessor has completed and its writes are visible (a no-op for a normal
// launch), and pdl_trigger() lets the successor start launching once every
// CTA of this grid has issued it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Distributed shared memory of a thread-block cluster (1-D clusters): this
// CTA's rank, the address of a shared variable of this CTA mapped to the same
// variable of CTA `rank`, plain loads through such an address, and the
// barrier over every thread of every CTA of the cluster (release / acquire,
// so shared-memory writes before it are visible to the cluster after it).
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ int ldc_s32(uint32_t a) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float ldc_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// launch_pdl with clusters of `cluster` CTAs along x (the grid a multiple).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_cluster_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      int cluster, cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// CTAs per sequence of the carry scans (phase B, bwd B): with few sequences
// a sequence's chunks are split over a cluster of G CTAs (G a power of two
// up to 8, G x sequences within the SM count, at least 64 chunks per CTA),
// so that more SMs share the scan.
inline int carry_scan_cluster(int64_t BH, int64_t C, int sms) {
    int G = 1;
    while (G < 8 && BH * 2 * G <= sms && C >= (int64_t)64 * 2 * G) G *= 2;
    return G;
}

// Warps per CTA for a chunk kernel with `per_warp` bytes of shared memory
// per warp: 4 or 8, whichever keeps more warps resident per SM by the
// runtime's occupancy calculation (registers, shared memory with the
// dictionary region paid once per CTA, and the per-SM limits).  Answers are
// cached per (kernel, shared-memory sizes).
struct WpcCacheEntry {
    const void *kern;
    int per_warp, dict_bytes, wpc;
};

template <typename KernT>
inline int choose_wpc(KernT kern, const ChunkParams &p, int per_warp) {
    static WpcCacheEntry cache[64];
    static int used = 0;
    static std::mutex mu;
    const void *key = reinterpret_cast<const void *>(kern);
    ChunkParams q = p;
    q.wpc = 4;
    const int dict4 = dict_region_bytes(q);
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].kern == key && cache[i].per_warp == per_warp &&
                cache[i].dict_bytes == dict4)
                return cache[i].wpc;
    }
    const int budget = 227 * 1024;
    int best = 4, best_warps = -1;
    for (int wpc = 4; wpc <= kMaxWPC; wpc *= 2) {
        q.wpc = wpc;
        const int smem = dict_region_bytes(q) + wpc * per_warp + 256;
        if (smem > budget) continue;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            continue;
        int blocks = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, wpc * 32, smem) !=
            cudaSuccess)
            continue;
        if (blocks * wpc >= best_warps) {
            best_warps = blocks * wpc;
            best = wpc;
        }
    }
    std::lock_guard<std::mutex> lock(mu);
    if (used < 64) cache[used++] = WpcCacheEntry{key, per_warp, dict4, best};
    return best;
}

template <typename KernT>
inline cudaError_t launch_units(KernT kern, ChunkParams p, int per_warp, cudaStream_t st,
                                bool pdl = false) {
    p.smem_per_warp = per_warp;
    p.wpc = choose_wpc(kern, p, per_warp);
    const size_t smem = (size_t)dict_region_bytes(p) + (size_t)p.wpc * per_warp + 256;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (p.units + p.wpc - 1) / p.wpc;
    if (pdl) return launch_pdl(kern, dim3((unsigned)grid), dim3(p.wpc * 32), smem, st, p);
    kern<<<(unsigned)grid, p.wpc * 32, smem, st>>>(p);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// host-side argument checks and error text (api.cu)
// ---------------------------------------------------------------------------
pdssm_status check_scan_dims(const pdssm_dims *dm, int64_t pi_hs, int64_t chunk);
pdssm_status cuda_fail(cudaError_t e, const char *where);   // sets the last-error text
pdssm_status arg_fail(pdssm_status st, const char *why);    // sets the last-error text

// ---------------------------------------------------------------------------
// host launchers (one per kernel family)
// ---------------------------------------------------------------------------
cudaError_t launch_select(const pdssm_dims &dm, const void *u, pdssm_dtype ut, const float *W,
                          int32_t *k_out, bool use_tc, float *logits_out, float *scale_out,
                          cudaStream_t st);
bool select_tc_supported(const pdssm_dims &dm, pdssm_dtype ut, const void *u, const float *W);
cudaError_t launch_select_tc(const pdssm_dims &dm, const void *u, const float *W, int32_t *k_out,
                             float *logits_out, float *scale_out, cudaStream_t st);
cudaError_t launch_prep(const pdssm_dims &dm, const int32_t *pi, int64_t pi_hs, int32_t *dict,
                        uint2 *seg, uint2 *segw, int *dict_stats,
                        uint8_t *tab, int32_t *fan, int64_t Hd, int *status, cudaStream_t st);
cudaError_t launch_validate(const pdssm_dims &dm, const int32_t *pi, int64_t pi_hs,
                            const int32_t *k, int *counts, cudaStream_t st);
cudaError_t launch_phaseA(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st);
bool fast_path(const ChunkParams &p);
cudaError_t launch_phaseA_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st);
cudaError_t launch_phaseC_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st);
cudaError_t launch_scan_fused(ChunkParams p, pdssm_dtype dt, cudaStream_t st, bool select);
bool fused_path(const ChunkParams &p);
bool fused_select_ok(const ChunkParams &p, const void *u, const float *W);
cudaError_t launch_wait_selftest(const ChunkParams &p, int which, cudaStream_t st);
cudaError_t launch_dict_hardmax(int64_t n_mats, int N, const float *A, int32_t *pi,
                                cudaStream_t st);
cudaError_t launch_soft_maps(const pdssm_dims &dm, const void *u, pdssm_dtype ut,
                             const float *W, const float *A, int64_t a_hs, float inv_tau,
                             int32_t *maps, cudaStream_t st);
size_t surrogate_scratch_bytes(const pdssm_dims &dm, int64_t a_hs);
cudaError_t launch_surrogate(const pdssm_dims &dm, const void *u, pdssm_dtype ut, const float *W,
                             const float *A, int64_t a_hs, const int32_t *pi, const int32_t *k,
                             const void *d, const void *b, pdssm_dtype dt, const float *h0,
                             const float *Hc, int64_t chunk, const float *lam, float inv_tau_s,
                             float inv_tau_a, void *scratch, float *g_l, float *g_W, float *g_A,
                             cudaStream_t st);
cudaError_t launch_scan_maps(const pdssm_dims &dm, const int32_t *maps, const void *d,
                             const void *b, const void *c, pdssm_dtype dt, const float *h0,
                             float *y, float *h_last, cudaStream_t st);
cudaError_t launch_bwdA_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st);
cudaError_t launch_bwdC_fast(ChunkParams p, pdssm_dtype dt, cudaStream_t st);
cudaError_t launch_phaseB(const ChunkParams &p, cudaStream_t st);
cudaError_t launch_phaseC(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st);
cudaError_t launch_bwdA(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st);
cudaError_t launch_bwdB(const ChunkParams &p, cudaStream_t st);
cudaError_t launch_bwdC(const ChunkParams &p, pdssm_dtype dt, cudaStream_t st);

}  // namespace pdssm
