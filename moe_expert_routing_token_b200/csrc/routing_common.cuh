// Device helpers shared by the routing kernels of libmoe_routing.
//
// Scoring follows the SGLang MoE routing page ("[SGLang] MoE 라우팅: 토큰에서
// 전문가로의 배분 알고리즘"): softmax over the row (§2, §3) or a per-expert
// sigmoid (§4).  All arithmetic is fp32.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

enum Scoring : int { kSoftmax = 0, kSigmoid = 1 };
enum GroupKind : int { kGroupMax = 0, kGroupTop2Sum = 1 };

constexpr unsigned kFullMask = 0xffffffffu;

// Kernel arguments (plain pointers and sizes; identical for every variant).
struct RouteArgs {
    const void* logits;   // (M, E) fp32 or bf16, row-major
    const float* bias;    // (E,) fp32 or nullptr
    int64_t M;
    int E;
    int G;                // num_expert_group
    int TG;               // topk_group
    int K;                // topk
    int group_kind;       // GroupKind
    int renorm;
    float rsf;            // routed_scaling_factor
    float* weights;       // (M, K) fp32
    int32_t* ids;         // (M, K) int32
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Logistic function in fp32: 1 / (1 + 2^(-x * log2(e))) with the hardware
// base-2 exponential and reciprocal approximations (ex2.approx.ftz,
// rcp.approx.ftz): one multiply, two MUFU operations and one add.  Absolute
// error is below 2e-7 for |x| <= 16 (checked against the double-precision
// oracle); for x < -87 the result underflows to 0 (subnormals flush to zero).
__device__ __forceinline__ float sigmoid_f32(float x) {
    const float t = x * -1.4426950408889634f;  // -x * log2(e)
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(t));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
    return r;
}

// e^x for the softmax: 2^(x * log2(e)) with the hardware approximation.
__device__ __forceinline__ float exp_f32(float x) {
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(x * 1.4426950408889634f));
    return e;
}

// Three-input max / min (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Total order on (score, index) pairs as one unsigned 64-bit key: a larger key
// means a larger score, or an equal score and a smaller index.  -0 is folded
// into +0 first so that the order matches float comparison.
__device__ __forceinline__ unsigned long long order_key(float v, int idx) {
    uint32_t f = __float_as_uint(v + 0.0f);
    f = (f & 0x80000000u) ? ~f : (f | 0x80000000u);
    return (static_cast<unsigned long long>(f) << 32) | static_cast<uint32_t>(~idx);
}
__device__ __forceinline__ int order_key_index(unsigned long long k) {
    return static_cast<int>(~static_cast<uint32_t>(k));
}

// a beats b: larger value, or equal value and smaller index.
__device__ __forceinline__ bool beats(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// Merge two (largest, second largest) pairs counting multiplicity.
__device__ __forceinline__ void top2_merge(float& a1, float& a2, float b1, float b2) {
    const float n2 = fmax3(fminf(a1, b1), a2, b2);
    a1 = fmaxf(a1, b1);
    a2 = n2;
}

__device__ __forceinline__ void top2_push(float& m1, float& m2, float v) {
    float t = fminf(m1, v);
    m1 = fmaxf(m1, v);
    m2 = fmaxf(m2, t);
}

// Largest and second largest (with multiplicity) of N values, N even, by a
// pairwise tree: N/2 (max, min) pairs, then N/2 - 1 merges.
template <int N>
__device__ __forceinline__ void top2_of(const float (&v)[N], float& m1, float& m2) {
    static_assert(N % 2 == 0, "even chunk");
    float h[N / 2], l[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        h[i] = fmaxf(v[2 * i], v[2 * i + 1]);
        l[i] = fminf(v[2 * i], v[2 * i + 1]);
    }
#pragma unroll
    for (int w = 1; w < N / 2; w *= 2) {
#pragma unroll
        for (int i = 0; i + w < N / 2; i += 2 * w) top2_merge(h[i], l[i], h[i + w], l[i + w]);
    }
    m1 = h[0];
    m2 = l[0];
}

template <typename T>
__device__ __forceinline__ float load_scalar(const T* p);
template <>
__device__ __forceinline__ float load_scalar<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_scalar<__nv_bfloat16>(const __nv_bfloat16* p) {
    unsigned short u = __ldg(reinterpret_cast<const unsigned short*>(p));
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

// Load N consecutive elements starting at p (p aligned to the widest vector
// that divides N * sizeof(T)) and widen them to fp32.
template <typename T, int N>
struct ChunkLoader;

template <int N>
struct ChunkLoader<float, N> {
    static_assert(N % 4 == 0, "fp32 chunks are loaded as float4");
    __device__ __forceinline__ static void load(const float* p, float (&x)[N]) {
        const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            float4 v = __ldg(q + i);
            x[4 * i + 0] = v.x;
            x[4 * i + 1] = v.y;
            x[4 * i + 2] = v.z;
            x[4 * i + 3] = v.w;
        }
    }
};

template <int N>
struct ChunkLoader<__nv_bfloat16, N> {
    static_assert(N % 4 == 0, "bf16 chunks are loaded as 8- or 16-byte vectors");
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&x)[N]) {
        if constexpr (N % 8 == 0) {
            const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
            for (int i = 0; i < N / 8; ++i) {
                uint4 v = __ldg(q + i);
                x[8 * i + 0] = bf16_lo(v.x);
                x[8 * i + 1] = bf16_hi(v.x);
                x[8 * i + 2] = bf16_lo(v.y);
                x[8 * i + 3] = bf16_hi(v.y);
                x[8 * i + 4] = bf16_lo(v.z);
                x[8 * i + 5] = bf16_hi(v.z);
                x[8 * i + 6] = bf16_lo(v.w);
                x[8 * i + 7] = bf16_hi(v.w);
            }
        } else {
            const uint2* q = reinterpret_cast<const uint2*>(p);
#pragma unroll
            for (int i = 0; i < N / 4; ++i) {
                uint2 v = __ldg(q + i);
                x[4 * i + 0] = bf16_lo(v.x);
                x[4 * i + 1] = bf16_hi(v.x);
                x[4 * i + 2] = bf16_lo(v.y);
                x[4 * i + 3] = bf16_hi(v.y);
            }
        }
    }
};

}  // namespace moe
