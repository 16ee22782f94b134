// Prefill path of the VQ-MoE layer (tcgen05 grouped GEMM): not built yet.
#include "vq_internal.h"

namespace vq {

size_t prefill_workspace_size(const vq_moe_layer *L, int T, int k)
{
    size_t o = 0;
    plan_routing(o, T, k, L->gate.E);
    return o;
}

vq_status run_prefill(const vq_moe_layer *, const uint16_t *, int, const float *, int, int, void *, int, void *,
                      size_t, cudaStream_t)
{
    return VQ_ERR_UNSUPPORTED;
}

}  // namespace vq
