// The fused top-1 router for small expert counts, on the CUDA cores: the
// CUDA-core kernel of the SGLang MoE routing page ("[SGLang] MoE 라우팅: 토큰에서
// 전문가로의 배분 알고리즘", §5 Fused MoE Router).  Per token row:
//
//   l_e  = sum_k h[k] * W(k, e)        bf16 inputs, fp32 accumulation
//   cap  = c * tanh(l / c)             the softcapping (c = 0: none)
//   id   = arg-max_e l_e               lowest index among equal logits
//   w    = 1 / sum_e exp(cap_e - cap_id)   the page's invsumexp
//
// The arg-max is taken on the raw logits.  c * tanh(x / c) is monotone, so
// the raw maximum is also a maximum of the capped values, but it is not
// injective in finite precision: far in the saturated range (|x / c| above
// about 9 in fp32, 19 in double) distinct logits cap to the same value.  Such
// a row has several equal largest capped values; the raw arg-max is one of
// them, and the weight, which depends only on the capped values, is the same
// whichever of them is chosen.
//
// This kernel serves the (K, E) weight layout and hidden sizes that are not
// a multiple of 64; the rest goes to the tensor-core kernel (top1_tc.cu).
// With E <= 8 experts the work is 2 * E flops per 2-byte hidden value, below
// the B200's fp32 CUDA-core ridge (about 11 flops per byte), but the
// instruction issue (the FMAs plus the bf16 unpacking) is close to the rate
// at which HBM delivers the hidden states at E = 8 (measured: 1.1 TB/s at
// M = 8192, against 4.9 TB/s for the tensor-core kernel).  Each 128-thread block takes
// 4 rows at a time; every thread walks 8-value chunks of the hidden size,
// loads the chunk's weights once (E 16-byte vectors, cached in L1/L2) and
// applies them to the 4 rows.  The partial sums meet through warp shuffles
// and then shared memory, in a fixed order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>

#include "moe_routing.h"
#include "routing_common.cuh"

namespace moe {

int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);
int sm_count(int* dev, int* sms);
int launch_top1_tc(const void* h, const void* w, int64_t M, int K, int E, float softcap, float* weights,
                   int32_t* ids, float* logits_out, cudaStream_t st);

namespace {

constexpr int kT1Threads = 128;
constexpr int kT1Warps = kT1Threads / 32;
constexpr int kT1Rows = 4;        // rows sharing each weight chunk
constexpr int kT1Chunk = 8;       // hidden values per 16-byte load
constexpr int kT1BlocksPerSm = 4;
constexpr int kT1MaxE = 8;
constexpr int kT1TcBlockK = 64;     // its k-block
constexpr int kT1TcMaxE = 256;      // UMMA N limit for M = 128

// The 8 bf16 values of a 16-byte vector, as fp32.
__device__ __forceinline__ void unpack8(const uint4 q, float (&x)[kT1Chunk]) {
    x[0] = bf16_lo(q.x);
    x[1] = bf16_hi(q.x);
    x[2] = bf16_lo(q.y);
    x[3] = bf16_hi(q.y);
    x[4] = bf16_lo(q.z);
    x[5] = bf16_hi(q.z);
    x[6] = bf16_lo(q.w);
    x[7] = bf16_hi(q.w);
}

// Weights of hidden values [8c, 8c + 8) for every expert: wf[t][e] = W(8c + t, e).
//   W_KE: W stored (K, E) row-major - the chunk is 8 * E contiguous values,
//         E 16-byte vectors (element j of the chunk is (t, e) = (j / E, j % E));
//   else: W stored (E, K) row-major - one 16-byte vector per expert row.
template <int E, bool W_KE>
__device__ __forceinline__ void load_weight_chunk(const __nv_bfloat16* __restrict__ w, int K, int c,
                                                  float (&wf)[kT1Chunk][E]) {
    if constexpr (W_KE) {
        const uint4* src = reinterpret_cast<const uint4*>(w + (int64_t)c * kT1Chunk * E);
#pragma unroll
        for (int v = 0; v < E; ++v) {
            float x[kT1Chunk];
            unpack8(__ldg(src + v), x);
#pragma unroll
            for (int j = 0; j < kT1Chunk; ++j) {
                const int flat = v * kT1Chunk + j;
                wf[flat / E][flat % E] = x[j];
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float x[kT1Chunk];
            unpack8(__ldg(reinterpret_cast<const uint4*>(w + (int64_t)e * K + (int64_t)c * kT1Chunk)), x);
#pragma unroll
            for (int t = 0; t < kT1Chunk; ++t) wf[t][e] = x[t];
        }
    }
}

template <int E, bool W_KE>
__global__ void __launch_bounds__(kT1Threads, kT1BlocksPerSm)
    top1_router_kernel(const __nv_bfloat16* __restrict__ h, const __nv_bfloat16* __restrict__ w, int64_t M,
                       int K, float softcap, float* __restrict__ weights, int32_t* __restrict__ ids,
                       float* __restrict__ logits_out) {
    __shared__ float s_part[kT1Warps][kT1Rows * E];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nchunks = K / kT1Chunk;
    const int64_t ntiles = (M + kT1Rows - 1) / kT1Rows;

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t row0 = tile * kT1Rows;
        const int rows = (int)((M - row0) < kT1Rows ? (M - row0) : kT1Rows);  // 1..4, same for the block
        float acc[kT1Rows][E];
#pragma unroll
        for (int r = 0; r < kT1Rows; ++r)
#pragma unroll
            for (int e = 0; e < E; ++e) acc[r][e] = 0.0f;

#pragma unroll 2
        for (int c = threadIdx.x; c < nchunks; c += kT1Threads) {
            float wf[kT1Chunk][E];
            load_weight_chunk<E, W_KE>(w, K, c, wf);
#pragma unroll
            for (int r = 0; r < kT1Rows; ++r) {
                if (r < rows) {
                    // hidden states are read once: stream them past L1
                    const uint4 q =
                        __ldcs(reinterpret_cast<const uint4*>(h + (row0 + r) * (int64_t)K + (int64_t)c * kT1Chunk));
                    float x[kT1Chunk];
                    unpack8(q, x);
#pragma unroll
                    for (int t = 0; t < kT1Chunk; ++t)
#pragma unroll
                        for (int e = 0; e < E; ++e) acc[r][e] = fmaf(x[t], wf[t][e], acc[r][e]);
                }
            }
        }

        // block sum of the partial logits: lanes, then warps in index order
#pragma unroll
        for (int r = 0; r < kT1Rows; ++r)
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float v = acc[r][e];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFullMask, v, off);
                if (lane == 0) s_part[warp][r * E + e] = v;
            }
        __syncthreads();

        if (threadIdx.x < rows) {
            const int r = threadIdx.x;
            const int64_t row = row0 + r;
            float l[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float s = s_part[0][r * E + e];
#pragma unroll
                for (int q = 1; q < kT1Warps; ++q) s += s_part[q][r * E + e];
                l[e] = s;
            }
            if (logits_out) {
#pragma unroll
                for (int e = 0; e < E; ++e) logits_out[row * E + e] = l[e];
            }
            int best = 0;
#pragma unroll
            for (int e = 1; e < E; ++e)
                if (l[e] > l[best]) best = e;
            float sum = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) sum += softmax_num(l[e], l[best], softcap);
            weights[row] = 1.0f / sum;
            ids[row] = best;
        }
        __syncthreads();  // s_part is rewritten by the next tile
    }
}

template <int E>
int launch_top1(bool w_ke, const void* h, const void* w, int64_t M, int K, float softcap, float* weights,
                int32_t* ids, float* logits_out, cudaStream_t st) {
    int dev = 0, sms = 0;
    const int rc = sm_count(&dev, &sms);
    if (rc != MOE_OK) return rc;
    const int64_t ntiles = (M + kT1Rows - 1) / kT1Rows;
    const int64_t cap = (int64_t)sms * kT1BlocksPerSm;
    const unsigned grid = (unsigned)(ntiles < cap ? ntiles : cap);
    const auto* hb = static_cast<const __nv_bfloat16*>(h);
    const auto* wb = static_cast<const __nv_bfloat16*>(w);
    if (w_ke)
        top1_router_kernel<E, true><<<grid, kT1Threads, 0, st>>>(hb, wb, M, K, softcap, weights, ids, logits_out);
    else
        top1_router_kernel<E, false><<<grid, kT1Threads, 0, st>>>(hb, wb, M, K, softcap, weights, ids, logits_out);
    const cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? MOE_OK : set_cuda_error(err, "moe_fused_router_top1: launch");
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_fused_router_top1(const void* hidden_states, const void* router_weight, int weight_layout, int64_t M,
                          int32_t K, int32_t E, float softcap, float* topk_weights, int32_t* topk_ids,
                          float* logits_out, void* stream) {
    using namespace moe;
    char msg[256];
    if (M < 0 || K < 1 || E < 1) {
        std::snprintf(msg, sizeof msg, "moe_fused_router_top1: bad sizes M=%lld K=%d E=%d", (long long)M, K, E);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (weight_layout != MOE_WEIGHT_K_BY_E && weight_layout != MOE_WEIGHT_E_BY_K) {
        std::snprintf(msg, sizeof msg, "moe_fused_router_top1: weight_layout %d is not MOE_WEIGHT_K_BY_E or "
                      "MOE_WEIGHT_E_BY_K", weight_layout);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (!(softcap == softcap) || softcap > 3.4e38f || softcap < -3.4e38f)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fused_router_top1: softcap is not finite");
    // The tensor-core kernel whenever K is a multiple of its 64-wide k-block,
    // the weights are (E, K) (K-major tiles) and E <= 256.  The page sends
    // batches below 512 tokens with E <= 8 to the CUDA cores; measured here
    // at M = 64, K = 7168 the CUDA-core kernel takes 13.7 us (E = 8) and the
    // tensor-core kernel 5.6 us (E = 16), so the CUDA-core kernel serves only
    // the (K, E) layout and K not a multiple of 64.
    const bool tc = K % kT1TcBlockK == 0 && weight_layout == MOE_WEIGHT_E_BY_K && E <= kT1TcMaxE;
    if (!tc && E > kT1MaxE) {
        std::snprintf(msg, sizeof msg,
                      "moe_fused_router_top1: E=%d needs the tensor-core kernel: (E, K) weights, K a multiple of "
                      "%d and E <= %d (got K=%d, layout %d); the CUDA-core kernel takes E <= %d",
                      E, kT1TcBlockK, kT1TcMaxE, K, weight_layout, kT1MaxE);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (!tc && K % kT1Chunk != 0) {
        std::snprintf(msg, sizeof msg, "moe_fused_router_top1: K=%d is not a multiple of %d", K, kT1Chunk);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (M == 0) return MOE_OK;
    if (!hidden_states || !router_weight || !topk_weights || !topk_ids)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fused_router_top1: null pointer argument");
    auto al = [](const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; };
    if (!al(hidden_states, 16) || !al(router_weight, 16) || !al(topk_weights, 4) || !al(topk_ids, 4) ||
        (logits_out && !al(logits_out, 4)))
        return set_error(MOE_ERR_INVALID_ARG,
                         "moe_fused_router_top1: hidden_states and router_weight must be 16-byte aligned, "
                         "outputs 4-byte aligned");
    const bool w_ke = weight_layout == MOE_WEIGHT_K_BY_E;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (tc) return launch_top1_tc(hidden_states, router_weight, M, K, E, softcap, topk_weights, topk_ids, logits_out, st);
    switch (E) {
        case 1: return launch_top1<1>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
        case 2: return launch_top1<2>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
        case 3: return launch_top1<3>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
        case 4: return launch_top1<4>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
        case 5: return launch_top1<5>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
        case 6: return launch_top1<6>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
        case 7: return launch_top1<7>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
        default: return launch_top1<8>(w_ke, hidden_states, router_weight, M, K, softcap, topk_weights, topk_ids, logits_out, st);
    }
}

}  // extern "C"
