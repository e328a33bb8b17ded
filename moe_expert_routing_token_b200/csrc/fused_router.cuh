// Fused router projection + routing (declarations shared with the C ABI layer).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "routing_common.cuh"

namespace moe {

// Helpers implemented in api.cu.
int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);
int sm_count(int* dev, int* sms);
int read_fused_watchdog(unsigned int* count);
// Barrier-wait timeouts of the tensor-core top-1 router (top1_tc.cu).
int read_top1_watchdog(unsigned int* count);
int route_logits(const void* logits, int dtype, const float* bias, int64_t M, int E, int K,
                 int renorm, int G, int TG, float rsf, float* weights, int32_t* ids, void* stream);

// Decode-sized batches of the fused router (fused_decode.cu): workspace bytes
// for the partial logits, the two launches, and their watchdog count.
size_t fused_decode_workspace_bytes(int64_t M, int num_kb);
int launch_fused_decode(const CUtensorMap& tmA, const void* router_weight, bool b_mn, const RouteArgs& route,
                        float* logits_out, int num_kb, void* workspace, cudaStream_t st);
int read_decode_watchdog(unsigned int* count);

}  // namespace moe
