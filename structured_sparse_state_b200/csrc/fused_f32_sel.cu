// Instantiation of the single-pass forward (fused.cuh) for fp32 rows, with
// the selection inside.
#include "fused.cuh"

namespace pdssm {

cudaError_t launch_fused_f32_sel(ChunkParams p, cudaStream_t st) {
    return p.N == 64 ? launch_fused_t<float, 2, true>(p, st)
                     : launch_fused_t<float, 1, true>(p, st);
}

}  // namespace pdssm
