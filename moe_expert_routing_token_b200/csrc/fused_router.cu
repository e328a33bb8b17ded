// Fused router: hidden_states x router_weight on the tensor cores, routing on
// the fp32 accumulator (SGLang MoE routing page, §5 Fused MoE Router).
#include "fused_router.cuh"
#include "moe_routing.h"

namespace moe {
int read_fused_watchdog(unsigned int* count) {
    *count = 0;
    return 0;
}
}  // namespace moe

extern "C" {

size_t moe_fused_router_workspace_size(int64_t M, int32_t K, int32_t E) {
    if (M < 0 || K < 1 || E < 1) return (size_t)-1;
    return 0;
}

int moe_fused_router_topk(const void* hidden_states, const void* router_weight, int weight_layout,
                          const float* correction_bias, int64_t M, int32_t K, int32_t E,
                          int32_t topk, int32_t renormalize, int32_t num_expert_group,
                          int32_t topk_group, float routed_scaling_factor, float* topk_weights,
                          int32_t* topk_ids, float* logits_out, void* workspace,
                          size_t workspace_bytes, void* stream) {
    (void)hidden_states; (void)router_weight; (void)weight_layout; (void)correction_bias;
    (void)M; (void)K; (void)E; (void)topk; (void)renormalize; (void)num_expert_group;
    (void)topk_group; (void)routed_scaling_factor; (void)topk_weights; (void)topk_ids;
    (void)logits_out; (void)workspace; (void)workspace_bytes; (void)stream;
    return moe::set_error(MOE_ERR_UNSUPPORTED, "moe_fused_router_topk: not built yet");
}

}  // extern "C"
