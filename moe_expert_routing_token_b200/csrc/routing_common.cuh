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
constexpr uint64_t kWaitBudgetNs = 2000000000ull;  // 2 s per barrier wait

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
    int bias_bf16 = 0;    // 1: round the bias to bf16 before use (the aiter variant)
    float softcap = 0.0f; // softmax: weights from c * tanh(x / c) (0: none)
    // Partial-logit input (fused router, decode batches): `logits` holds
    // nparts fp32 partial sums, part_stride floats apart, added in order.
    int nparts = 0;
    int64_t part_stride = 0;
    float* logits_out = nullptr;  // (M, E) fp32 copy of the summed logits, or nullptr
};



// The correction bias as the kernels use it: fp32, or (aiter variant, bf16
// logits) rounded to the logits dtype first.
__device__ __forceinline__ float bias_as_used(float b, int round_bf16) {
    return round_bf16 ? __bfloat162float(__float2bfloat16_rn(b)) : b;
}

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

// Packed fp32 pairs (sm_100 paired FADD/FMUL).
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
    return (static_cast<unsigned long long>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float lo2(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(unsigned long long v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Smallest logit the pair sigmoid accepts: 1 + 2^(43.5 log2 e) stays below
// 2^63, so the product of two denominators cannot overflow.  sigmoid(-43.5)
// is 1.3e-19; clamping lower logits to it moves a score by less than that.
constexpr float kSigmoidClamp = -43.5f;
constexpr uint32_t kSigmoidClampBf16x2 = 0xC22EC22Eu;  // bf16 -43.5 in both halves

// Logistic function of two values with one reciprocal:
// 1/d0 = d1 * rcp(d0 d1), 1/d1 = d0 * rcp(d0 d1), d = 1 + 2^(-x log2 e).
// Inputs must be >= kSigmoidClamp.  Relative error ~3e-7; used for the
// selection keys (the weights use sigmoid_f32 on the raw logit).
__device__ __forceinline__ unsigned long long sigmoid_pair(unsigned long long x) {
    const unsigned long long t = mul2(x, pack2(-1.4426950408889634f, -1.4426950408889634f));
    float e0, e1, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(lo2(t)));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(hi2(t)));
    const unsigned long long d = add2(pack2(e0, e1), pack2(1.0f, 1.0f));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(lo2(d) * hi2(d)));
    return mul2(pack2(hi2(d), lo2(d)), pack2(r, r));
}

__device__ __forceinline__ uint32_t clamp_bf16x2_for_sigmoid(uint32_t w) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(kSigmoidClampBf16x2));
    return r;
}

// e^x for the softmax: 2^(x * log2(e)) with the hardware approximation.
__device__ __forceinline__ float exp_f32(float x) {
    float e;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(x * 1.4426950408889634f));
    return e;
}

// Logit softcapping of the fused router (routing page §5): c * tanh(x / c),
// with the accurate tanhf; c = 0 leaves x as it is.  It is monotone, so the
// experts chosen on the raw logits are also the best by capped value; only
// the softmax weights and denominators use the capped values.  It is not
// injective in finite precision: deep in saturation distinct logits cap to
// one value, and the raw order then picks one member of that tie set.
__device__ __forceinline__ float softcap_f32(float x, float c) { return c != 0.0f ? c * tanhf(x / c) : x; }

// exp(cap(v) - cap(vmax)), the softmax numerator relative to the row max.
__device__ __forceinline__ float softmax_num(float v, float vmax, float c) {
    return exp_f32(softcap_f32(v, c) - softcap_f32(vmax, c));
}

// Bound on |tanh.approx.f32(y) - tanh(y)| used to size the approximate-key
// band: four times the instruction's documented maximum error of about 2^-11,
// and checked exhaustively for every bf16 input on the device by the tests.
constexpr float kTanhApproxErr = 1.0f / 512.0f;
// Bound on the difference between the paired-reciprocal and the single
// sigmoid keys (a few fp32 ulp of values below 2).
constexpr float kPairKeyErr = 1.0f / 1048576.0f;

__device__ __forceinline__ float tanh_approx(float y) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(y));
    return r;
}

__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Orderable unsigned key of a score: larger score, larger key.  NaN maps to
// 1, below every number, and 0 is left for empty slots.
__device__ __forceinline__ uint32_t order_u32(float v) {
    uint32_t f = __float_as_uint(v + 0.0f);
    f = (f & 0x80000000u) ? ~f : (f | 0x80000000u);
    return (v == v) ? f : 1u;
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

// Compare-exchange for descending order.
__device__ __forceinline__ void cx_desc(float& a, float& b) {
    const float hi = fmaxf(a, b);
    b = fminf(a, b);
    a = hi;
}

// Sort a bitonic sequence of N (power of two) values into descending order.
template <int N>
__device__ __forceinline__ void bitonic_clean_desc(float (&x)[N]) {
#pragma unroll
    for (int k = N / 2; k >= 1; k >>= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            if ((i & k) == 0) cx_desc(x[i], x[i + k]);
    }
}

// Over the aligned segment of L lanes, each lane contributing its sorted
// pair (v1 >= v2), return in every lane the 8 largest of the 2L values,
// descending (padded with -inf when 2L < 8).  Log2(L) xor-shuffle steps, each
// merging two sorted lists with a bitonic network.
template <int L>
__device__ __forceinline__ void segment_top8(float v1, float v2, float (&out)[8]) {
    float a[8] = {v1, v2, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
    if constexpr (L >= 2) {  // two sorted pairs -> sorted 4
        const float b0 = __shfl_xor_sync(kFullMask, a[0], 1);
        const float b1 = __shfl_xor_sync(kFullMask, a[1], 1);
        float y[4] = {a[0], a[1], b1, b0};
        bitonic_clean_desc(y);
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = y[i];
    }
    if constexpr (L >= 4) {  // two sorted 4-lists -> sorted 8
        float x[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[i] = a[i];
            x[7 - i] = __shfl_xor_sync(kFullMask, a[i], 2);
        }
        bitonic_clean_desc(x);
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = x[i];
    }
#pragma unroll
    for (int o = 4; o < L; o <<= 1) {  // two sorted 8-lists -> top 8
        float b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = __shfl_xor_sync(kFullMask, a[i], o);
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fmaxf(a[i], b[7 - i]);
        bitonic_clean_desc(a);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = a[i];
}

// The K-th largest (1 <= K <= 8) of a descending list: the minimum of its
// first K entries (no dynamically indexed array, which would go to local
// memory).
__device__ __forceinline__ float kth_of_sorted8(const float (&top)[8], int K) {
    float t = top[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) t = (i < K) ? fminf(t, top[i]) : t;
    return t;
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
