// tcgen05 / TMEM / TMA split-KV attention for sm_100a (B200).
#include "tpla_internal.cuh"

namespace tpla {

bool sm100_supports(const Plan&) { return false; }

cudaError_t launch_attention_sm100(const Plan&, const __nv_bfloat16*, const __nv_bfloat16*,
                                   const __nv_bfloat16*, const __nv_bfloat16*, const int32_t*,
                                   const int32_t*, Workspace, int, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace tpla
