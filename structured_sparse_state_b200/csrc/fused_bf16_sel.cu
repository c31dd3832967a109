// Instantiation of the single-pass forward (fused.cuh) for bf16 rows, with
// the selection inside.
#include "fused.cuh"

namespace pdssm {

cudaError_t launch_fused_bf16_sel(ChunkParams p, cudaStream_t st) {
    return p.N == 64 ? launch_fused_t<__nv_bfloat16, 2, true>(p, st)
                     : launch_fused_t<__nv_bfloat16, 1, true>(p, st);
}

}  // namespace pdssm
