// Fused router projection + routing (declarations shared with the C ABI layer).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Helpers implemented in api.cu.
int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);
int sm_count(int* dev, int* sms);
int read_fused_watchdog(unsigned int* count);
int route_logits(const void* logits, int dtype, const float* bias, int64_t M, int E, int K,
                 int renorm, int G, int TG, float rsf, float* weights, int32_t* ids, void* stream);

}  // namespace moe
