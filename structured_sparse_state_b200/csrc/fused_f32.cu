// Instantiation of the single-pass forward (fused.cuh) for fp32 rows.
#include "fused.cuh"

namespace pdssm {

cudaError_t launch_fused_f32(ChunkParams p, cudaStream_t st) {
    return p.N == 64 ? launch_fused_t<float, 2, false>(p, st)
                     : launch_fused_t<float, 1, false>(p, st);
}

}  // namespace pdssm
