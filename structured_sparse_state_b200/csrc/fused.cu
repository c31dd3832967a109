// Dispatch of the single-pass forward (fused.cuh).
#include "fused.cuh"

namespace pdssm {

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

cudaError_t launch_scan_fused(ChunkParams p, pdssm_dtype dt, cudaStream_t st, bool select) {
    const int es = dt == PDSSM_BF16 ? 2 : 4;
    p.dict_content = (dt == PDSSM_BF16 ? kDictMap16 : kDictMap) | kDictSeg;
    p.smem_per_warp = warp_smem_bytes(kFastStages, 3, (int)p.N * es);
    if (dt == PDSSM_BF16) return select ? launch_fused_bf16_sel(p, st) : launch_fused_bf16(p, st);
    return select ? launch_fused_f32_sel(p, st) : launch_fused_f32(p, st);
}

}  // namespace pdssm
