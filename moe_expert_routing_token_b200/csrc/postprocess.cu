// Post-processing of a finished routing result (topk_weights fp32 (M, k),
// topk_ids int32 (M, k)), in place:
//
//  * moe_fill_shared_expert_slot - the shared-expert slot of the SGLang MoE
//    routing page (§6 공유 전문가 슬롯 할당): the last slot of every row becomes
//    the shared expert E + pick[row] (pick: the random draw, in
//    [0, num_shared), supplied by the caller) and, when a routed scaling
//    factor is given, its weight becomes the sum of the row's other k-1
//    weights divided by that factor.
//  * moe_fill_shared_expert_slot_philox - the same slot with the draw made
//    here from a seed: Philox4x64-10 (Salmon et al., SC'11, "Parallel random
//    numbers: as easy as 1, 2, 3"), word 0 of the block at counter offset +
//    row under key (seed, 0), mapped to [0, num_shared) by the high word of
//    its product with num_shared.
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

// Word 0 of Philox4x64-10 for counter (c0, c1, 0, 0) and key (k0, 0): ten
// rounds, each multiplying words 0 and 2 by the generator's two constants
// (64 x 64 -> 128 bits), the key advanced by its two Weyl constants between
// rounds.
__device__ __forceinline__ uint64_t philox4x64_word0(uint64_t c0, uint64_t c1, uint64_t k0) {
    constexpr uint64_t kMul0 = 0xD2E7470EE14C6C93ull, kMul1 = 0xCA5A826395121157ull;
    constexpr uint64_t kWeyl0 = 0x9E3779B97F4A7C15ull, kWeyl1 = 0xBB67AE8584CAA73Bull;
    uint64_t x0 = c0, x1 = c1, x2 = 0, x3 = 0, k1 = 0;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += kWeyl0;
            k1 += kWeyl1;
        }
        const uint64_t hi0 = __umul64hi(kMul0, x0), lo0 = kMul0 * x0;
        const uint64_t hi1 = __umul64hi(kMul1, x2), lo1 = kMul1 * x2;
        const uint64_t y0 = hi1 ^ x1 ^ k0, y2 = hi0 ^ x3 ^ k1;
        x1 = lo1;
        x3 = lo0;
        x0 = y0;
        x2 = y2;
    }
    return x0;
}

__global__ void __launch_bounds__(kPostThreads)
    fill_shared_philox_kernel(float* __restrict__ w, int32_t* __restrict__ ids, int64_t M, int k, int E,
                              int num_shared, uint64_t seed, uint64_t offset, float rsf) {
    const int64_t row = (int64_t)blockIdx.x * kPostThreads + threadIdx.x;
    if (row >= M) return;
    const uint64_t c0 = offset + (uint64_t)row;
    const uint64_t u = philox4x64_word0(c0, c0 < offset ? 1ull : 0ull, seed);
    const int pick = (int)__umul64hi(u, (uint64_t)num_shared);
    int32_t* id = ids + row * k;
    float* wr = w + row * k;
    id[k - 1] = E + pick;
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

int moe_fill_shared_expert_slot_philox(float* topk_weights, int32_t* topk_ids, int64_t M, int32_t k, int32_t E,
                                       int32_t num_shared, uint64_t seed, uint64_t offset,
                                       float routed_scaling_factor, void* stream) {
    using namespace moe;
    const char* who = "moe_fill_shared_expert_slot_philox";
    int rc = check_result_args(who, topk_weights, topk_ids, M, k);
    if (rc != MOE_OK) return rc;
    if (E < 1 || num_shared < 1 || (int64_t)E + num_shared > INT32_MAX)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fill_shared_expert_slot_philox: bad E or num_shared");
    if (routed_scaling_factor != routed_scaling_factor)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fill_shared_expert_slot_philox: routed_scaling_factor is NaN");
    if (M == 0) return MOE_OK;
    fill_shared_philox_kernel<<<grid_for(M), kPostThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        topk_weights, topk_ids, M, k, E, num_shared, seed, offset, routed_scaling_factor);
    const cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? MOE_OK : set_cuda_error(err, who);
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
