// Forward phases A and C (three-phase forward) for a state that fills the
// warp (N = 32 or 64) with 16-byte aligned rows, on the segment routines
// of fwd_segments.cuh, and the bounded-wait self-test.  The general kernels
// in fwd.cu serve every other N and unaligned rows.
#include "fused.cuh"   // the look-back of the bounded-wait self-test
#include "fwd_segments.cuh"

namespace pdssm {

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

}  // namespace pdssm
