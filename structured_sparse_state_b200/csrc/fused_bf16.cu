// Instantiation of the single-pass forward (fused.cuh) for bf16 rows.
#include "fused.cuh"

namespace pdssm {

cudaError_t launch_fused_bf16(ChunkParams p, cudaStream_t st) {
    return p.N == 64 ? launch_fused_t<__nv_bfloat16, 2, false>(p, st)
                     : launch_fused_t<__nv_bfloat16, 1, false>(p, st);
}

}  // namespace pdssm
