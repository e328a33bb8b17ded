// Post-processing of a finished routing result (topk_weights fp32 (M, k),
// topk_ids int32 (M, k)), in place:
//
//  * moe_fill_shared_expert_slot - the shared-expert slot of the SGLang MoE
//    routing page (§6 공유 전문가 슬롯 할당): the last slot of every row becomes
//    the shared expert E + pick[row] (pick: the random draw, in
//    [0, num_shared), supplied by the caller) and, when a routed scaling
//    factor is given, its weight becomes the sum of the row's other k-1
//    weights divided by that factor.
//  * moe_sort_topk_by_id - ascending-id output (the MiniMax-M3 attention
//    page's minimax_decode_topk, 코드 분석 §1, sorts its top-k block ids):
//    each row's (weight, id) pairs reordered by ascending id, equal ids
//    keeping their order.
//
// Both are one thread per row; they move k * 8 bytes per row and are bound
// by launch latency at the routing batch sizes.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>

#include "moe_routing.h"

namespace moe {

int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);

namespace {

constexpr int kPostThreads = 128;
constexpr int kMaxK = 32;
constexpr int kRowStride = kMaxK + 1;  // odd word stride: one row per bank

__global__ void __launch_bounds__(kPostThreads)
    fill_shared_kernel(float* __restrict__ w, int32_t* __restrict__ ids, int64_t M, int k, int E,
                       const int32_t* __restrict__ pick, float rsf) {
    const int64_t row = (int64_t)blockIdx.x * kPostThreads + threadIdx.x;
    if (row >= M) return;
    int32_t* id = ids + row * k;
    float* wr = w + row * k;
    id[k - 1] = E + __ldg(pick + row);
    if (rsf != 0.0f) {
        float s = 0.0f;
        for (int j = 0; j < k - 1; ++j) s += wr[j];
        wr[k - 1] = s / rsf;
    }
}

__global__ void __launch_bounds__(kPostThreads)
    sort_by_id_kernel(float* __restrict__ w, int32_t* __restrict__ ids, int64_t M, int k) {
    __shared__ int32_t s_id[kPostThreads * kRowStride];
    __shared__ float s_w[kPostThreads * kRowStride];
    const int64_t row = (int64_t)blockIdx.x * kPostThreads + threadIdx.x;
    if (row >= M) return;
    int32_t* sid = s_id + threadIdx.x * kRowStride;
    float* sw = s_w + threadIdx.x * kRowStride;
    for (int j = 0; j < k; ++j) {
        sid[j] = ids[row * k + j];
        sw[j] = w[row * k + j];
    }
    for (int a = 1; a < k; ++a) {  // insertion sort: stable
        const int32_t ka = sid[a];
        const float wa = sw[a];
        int b = a - 1;
        while (b >= 0 && sid[b] > ka) {
            sid[b + 1] = sid[b];
            sw[b + 1] = sw[b];
            --b;
        }
        sid[b + 1] = ka;
        sw[b + 1] = wa;
    }
    for (int j = 0; j < k; ++j) {
        ids[row * k + j] = sid[j];
        w[row * k + j] = sw[j];
    }
}

int check_result_args(const char* who, const float* w, const int32_t* ids, int64_t M, int32_t k) {
    char msg[200];
    if (M < 0 || k < 1) {
        std::snprintf(msg, sizeof msg, "%s: bad sizes M=%lld k=%d", who, (long long)M, k);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (k > kMaxK) {
        std::snprintf(msg, sizeof msg, "%s: k=%d > %d", who, k, kMaxK);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (M > 0 && (!w || !ids)) {
        std::snprintf(msg, sizeof msg, "%s: null pointer argument", who);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    return MOE_OK;
}

unsigned grid_for(int64_t M) { return (unsigned)((M + kPostThreads - 1) / kPostThreads); }

}  // namespace
}  // namespace moe

extern "C" {

int moe_fill_shared_expert_slot(float* topk_weights, int32_t* topk_ids, int64_t M, int32_t k, int32_t E,
                                int32_t num_shared, const int32_t* shared_pick, float routed_scaling_factor,
                                void* stream) {
    using namespace moe;
    int rc = check_result_args("moe_fill_shared_expert_slot", topk_weights, topk_ids, M, k);
    if (rc != MOE_OK) return rc;
    if (E < 1 || num_shared < 1 || (int64_t)E + num_shared > INT32_MAX)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fill_shared_expert_slot: bad E or num_shared");
    if (routed_scaling_factor != routed_scaling_factor)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fill_shared_expert_slot: routed_scaling_factor is NaN");
    if (M == 0) return MOE_OK;
    if (!shared_pick) return set_error(MOE_ERR_INVALID_ARG, "moe_fill_shared_expert_slot: null shared_pick");
    fill_shared_kernel<<<grid_for(M), kPostThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        topk_weights, topk_ids, M, k, E, shared_pick, routed_scaling_factor);
    const cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? MOE_OK : set_cuda_error(err, "moe_fill_shared_expert_slot: launch");
}

int moe_sort_topk_by_id(float* topk_weights, int32_t* topk_ids, int64_t M, int32_t k, void* stream) {
    using namespace moe;
    int rc = check_result_args("moe_sort_topk_by_id", topk_weights, topk_ids, M, k);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    sort_by_id_kernel<<<grid_for(M), kPostThreads, 0, static_cast<cudaStream_t>(stream)>>>(topk_weights,
                                                                                         topk_ids, M, k);
    const cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? MOE_OK : set_cuda_error(err, "moe_sort_topk_by_id: launch");
}

}  // extern "C"
