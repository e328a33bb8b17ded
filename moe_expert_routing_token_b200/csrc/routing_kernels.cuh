// Routing kernels: logits (M, E) -> topk_weights (M, K) fp32, topk_ids (M, K) int32.
//
// What they compute is the routing of the SGLang MoE routing page
// ("[SGLang] MoE 라우팅: 토큰에서 전문가로의 배분 알고리즘"): §2 softmax top-k,
// §3 grouped top-k (group score = max) and §4 biased grouped top-k (sigmoid +
// correction_bias, group score = sum of the top-2 biased scores), with the
// gathered weights being the unbiased scores, renormalised and scaled.  Ties
// go to the lower expert / group index and ids leave in descending score.
//
// This file holds the SegRouter routing body and three kernels (the
// streaming kernels for large batches are in routing_stream.cuh, k <= 8, and
// routing_staged.cuh, k > 8):
//
//  * route_segment_kernel (E = 160 or 256, batches below 1024 rows): a row is
//    owned by a segment of L = E / C lanes, each lane holding C consecutive
//    experts in registers after one pass of 16-byte loads.  A lane's chunk
//    never straddles a group, so group scores need only xor-shuffles among
//    the group's lanes.  Instead of k rounds of arg-max, the kernel derives a
//    threshold tau that the k-th best admissible score is known to reach (for
//    k <= 8 the k-th largest of the kept lanes' top-2 values: they are k
//    distinct admissible experts), collects the few candidates >= tau into
//    shared memory, and ranks each candidate by counting how many candidates
//    beat it - the ballot/popcount rank idea of the MiniMax-M3 page's warp
//    rank sort, applied to scores.  Rows with more than kCandCap candidates
//    (massive ties) take an exact k-round arg-max.
//  * route_small_kernel (E <= 32): one thread per row, k rounds of arg-max in
//    registers.
//  * route_generic_kernel (any E <= 1024, any group shape, any alignment): one
//    warp per row, row staged in shared memory, k rounds of warp arg-max.
#pragma once

#include "routing_common.cuh"
#include "routing_threshold.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kSegThreads = 128;
constexpr int kCandCap = 32;
constexpr int kCandStride = kCandCap + 4;  // room for sentinels to a multiple of 4; 16-B rows

__device__ __forceinline__ unsigned seg_bits(int L) { return L >= 32 ? kFullMask : ((1u << L) - 1u); }

// Per-warp routing of R rows, L lanes per row, C consecutive experts per lane.
// `xin` holds the lane's C logits (fp32); everything after the load - scoring,
// group selection, candidate ranking, weights and the output stores - is here
// so that the standalone routing kernel and the fused router's epilogue run
// the same code.  `s_bias` is the correction bias in shared memory in the
// padded lane-chunk layout written by load_bias_padded() (ignored without
// BIAS): chunk j (experts [jC, jC+C)) starts at float j*CS, CS an odd number
// of float4, so the 16-byte reads of the L lanes of a segment hit distinct
// banks.
template <int E, int C, int SCORE, bool BIAS>
struct SegRouter {
    static constexpr int L = E / C;   // lanes per row
    static constexpr int R = 32 / L;  // rows per warp
    static constexpr int CQ = (C / 4) | 1;  // odd number of float4 per lane: conflict-free STS.128
    static constexpr int CS = CQ * 4;
    static constexpr int TPL = (32 + L - 1) / L;  // output ranks per lane (k <= 32)
    static_assert(E % C == 0 && 32 % L == 0 && C % 4 == 0 && C <= 32, "bad segment shape");

    static constexpr int BIAS_FLOATS = L * CS;  // padded bias layout

    struct Scratch {                            // one per warp; rows padded against bank conflicts
        float keys[R * L * CS];                 // selection keys of pass 1 (lane-chunk layout)
        unsigned long long cand[R][kCandStride];  // candidate order keys (+ zero sentinels)
        float2 out[R][33];                      // by rank: (unbiased score, id)
    };

    // Raw logits kept in a per-warp shared buffer (for callers whose logits
    // are not in shared memory); get() returns the unbiased score.
    struct StoredScores {
        float* warp_x;  // R * L * CS floats
        __device__ __forceinline__ void store(int q, float x0, float x1, float x2, float x3) const {
            const int lane = threadIdx.x & 31;
            reinterpret_cast<float4*>(warp_x + (lane / L * L + lane % L) * CS)[q] = make_float4(x0, x1, x2, x3);
        }
        __device__ __forceinline__ float get(int seg, int e) const {
            const float x = warp_x[(seg * L + e / C) * CS + e % C];
            return SCORE == kSigmoid ? sigmoid_f32(x) : x;
        }
    };

    // Copy the (E,) bias from global memory into the padded layout; called
    // by every thread of the block, followed by a barrier.
    __device__ __forceinline__ static void load_bias_padded(const float* g_bias, float* s_bias, int round_bf16) {
        for (int e = threadIdx.x; e < E; e += blockDim.x)
            s_bias[(e / C) * CS + e % C] = bias_as_used(__ldg(g_bias + e), round_bf16);
    }

    // Unbiased scores kept in a per-warp shared buffer (for callers whose raw
    // logits are not in shared memory).
    // XCLAMPED: the caller already raised sigmoid inputs to kSigmoidClamp.
    template <bool XCLAMPED = false, class PSrc>
    __device__ __forceinline__ static void route(const float (&xin)[C], bool valid, int64_t row,
                                                 const float* s_bias, Scratch& sc, const RouteArgs& a,
                                                 const PSrc& psrc) {
        const int lane = threadIdx.x & 31;
        const int seg = lane / L;
        const int sl = lane % L;
        const int base = seg * L;
        const int e0 = sl * C;
        const int G = a.G, TG = a.TG, K = a.K;
        const int P = L / G;  // lanes per group (the dispatcher guarantees G | L)
        const int g = sl / P;
        const bool all_groups = (TG == G);
        const int nsel_lanes = all_groups ? L : TG * P;
        const int need = (K + 1) >> 1;
        const unsigned smask = seg_bits(L) << base;
        float* my_keys = &sc.keys[(seg * L + sl) * CS];

        // Pass 1: score, selection key, per-lane top-2 of the keys.
        float key[C];
#pragma unroll
        for (int q = 0; q < C / 4; ++q) {
            psrc.store(q, xin[4 * q], xin[4 * q + 1], xin[4 * q + 2], xin[4 * q + 3]);
            float4 b = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if constexpr (BIAS) b = reinterpret_cast<const float4*>(s_bias + sl * CS)[q];
            unsigned long long k01, k23;
            if constexpr (SCORE == kSigmoid) {
                float x0 = xin[4 * q], x1 = xin[4 * q + 1], x2 = xin[4 * q + 2], x3 = xin[4 * q + 3];
                if constexpr (!XCLAMPED) {
                    x0 = fmaxf(x0, kSigmoidClamp);
                    x1 = fmaxf(x1, kSigmoidClamp);
                    x2 = fmaxf(x2, kSigmoidClamp);
                    x3 = fmaxf(x3, kSigmoidClamp);
                }
                k01 = sigmoid_pair(pack2(x0, x1));
                k23 = sigmoid_pair(pack2(x2, x3));
            } else {
                k01 = pack2(xin[4 * q], xin[4 * q + 1]);
                k23 = pack2(xin[4 * q + 2], xin[4 * q + 3]);
            }
            if constexpr (BIAS) {
                k01 = add2(k01, pack2(b.x, b.y));
                k23 = add2(k23, pack2(b.z, b.w));
            }
            key[4 * q + 0] = lo2(k01);
            key[4 * q + 1] = hi2(k01);
            key[4 * q + 2] = lo2(k23);
            key[4 * q + 3] = hi2(k23);
            reinterpret_cast<float4*>(my_keys)[q] =
                make_float4(key[4 * q], key[4 * q + 1], key[4 * q + 2], key[4 * q + 3]);
        }
        float m1, m2;
        top2_of(key, m1, m2);

        // Group score from the group's lanes, then keep the TG best groups
        // (nothing to do when every group is kept).
        bool gsel = true;
        if (!all_groups) {
            float g1 = m1, g2 = m2;
            for (int o = 1; o < P; o <<= 1) {
                const float b1 = __shfl_xor_sync(kFullMask, g1, o);
                const float b2 = __shfl_xor_sync(kFullMask, g2, o);
                top2_merge(g1, g2, b1, b2);
            }
            const float gs = (a.group_kind == kGroupTop2Sum) ? g1 + g2 : g1;
            int rank = 0;
            for (int h = 0; h < G; ++h) {
                const float o = __shfl_sync(kFullMask, gs, base + h * P);
                rank += (o > gs) || (o == gs && h < g);
            }
            gsel = rank < TG;
        }

        // Threshold: the kept lanes with the `need` largest second-best keys
        // hold at least K admissible experts with key >= tau.
        float tau;
        if (need > nsel_lanes) {
            tau = -INFINITY;
        } else if (need == nsel_lanes) {
            float v = gsel ? m2 : INFINITY;
#pragma unroll
            for (int o = L / 2; o >= 1; o >>= 1) v = fminf(v, __shfl_xor_sync(kFullMask, v, o));
            tau = v;
        } else if (K <= 8) {
            // Tighter: the K-th largest of all kept lanes' top-2 values (those
            // are K distinct kept experts).
            if constexpr (L == 8) {
                float vmax;
                tau = row_kth2<L>(gsel ? m1 : -INFINITY, gsel ? m2 : -INFINITY, K, vmax);
            } else {
                float top[8];
                segment_top8<L>(gsel ? m1 : -INFINITY, gsel ? m2 : -INFINITY, top);
                tau = kth_of_sorted8(top, K);
            }
        } else {
            const float my = gsel ? m2 : -INFINITY;
            int r = 0;
#pragma unroll
            for (int j = 0; j < L; ++j) {
                const float o = __shfl_sync(kFullMask, my, base + j);
                r += (o > my) || (o == my && j < sl);
            }
            const unsigned bal = __ballot_sync(kFullMask, r == need - 1) & smask;
            tau = __shfl_sync(kFullMask, my, __ffs(bal) - 1);
        }

        // Candidates: kept experts with key >= tau.
        unsigned mask = 0u;
        if (gsel) {
#pragma unroll
            for (int i = 0; i < C; ++i)
                if (key[i] >= tau) mask |= 1u << i;
        }
        // Inclusive prefix of the per-lane counts over the segment; its last
        // lane holds the segment total n.
        const int cnt = __popc(mask);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < L; o <<= 1) {
            const int t = __shfl_up_sync(kFullMask, incl, o);
            if (sl >= o) incl += t;
        }
        const int n = __shfl_sync(kFullMask, incl, base + L - 1);

        const bool exact_needed = valid && (n > kCandCap || n < K);
        if (__any_sync(kFullMask, exact_needed)) {
            // Exact K rounds of segment arg-max (massive ties; rare).
            unsigned taken = 0u;
            for (int j = 0; j < K; ++j) {
                int bi = -1;
                float bv = -INFINITY;
                if (gsel) {
#pragma unroll
                    for (int i = 0; i < C; ++i)
                        if (!((taken >> i) & 1u) && (bi < 0 || key[i] > bv)) {
                            bv = key[i];
                            bi = i;
                        }
                }
                float wv = bi < 0 ? -INFINITY : bv;
                int wi = bi < 0 ? 0x7fffffff : e0 + bi;
#pragma unroll
                for (int o = L / 2; o >= 1; o >>= 1) {
                    const float ov = __shfl_xor_sync(kFullMask, wv, o);
                    const int oi = __shfl_xor_sync(kFullMask, wi, o);
                    if (beats(ov, oi, wv, wi)) {
                        wv = ov;
                        wi = oi;
                    }
                }
                if (bi >= 0 && wi == e0 + bi) taken |= 1u << bi;
                if (sl == 0) {
                    const int gi = (wi >= 0 && wi < E) ? wi : 0;
                    sc.out[seg][j] = make_float2(psrc.get(seg, gi), __int_as_float(gi));
                }
            }
            __syncwarp();
        } else {
            // Compact the candidates of the segment into shared memory ...
            int pos = incl - cnt;
            unsigned mm = valid ? mask : 0u;
            while (mm) {
                const int b = __ffs(mm) - 1;
                mm &= mm - 1u;
                sc.cand[seg][pos] = order_key(my_keys[b], e0 + b);
                ++pos;
            }
            // zero keys pad the list to a multiple of 4 (they beat nothing)
            const int nn = valid ? n : 0;
            const int n4 = (nn + 3) & ~3;
            if (sl == 0)
                for (int u = nn; u < n4; ++u) sc.cand[seg][u] = 0ull;
            __syncwarp();
            // ... and rank each one by counting the candidates that beat it
            // (a lane takes candidates sl and sl + L in one pass).
            for (int t = sl; t < nn; t += 2 * L) {
                const int t2 = t + L;
                const unsigned long long c0 = sc.cand[seg][t];
                const unsigned long long c1 = t2 < nn ? sc.cand[seg][t2] : ~0ull;
                int r0 = 0, r1 = 0;
                for (int u = 0; u < n4; u += 4) {
                    const ulonglong2 d01 = *reinterpret_cast<const ulonglong2*>(&sc.cand[seg][u]);
                    const ulonglong2 d23 = *reinterpret_cast<const ulonglong2*>(&sc.cand[seg][u + 2]);
                    r0 += (d01.x > c0) + (d01.y > c0) + (d23.x > c0) + (d23.y > c0);
                    r1 += (d01.x > c1) + (d01.y > c1) + (d23.x > c1) + (d23.y > c1);
                }
                if (r0 < K) {
                    const int id = order_key_index(c0);
                    sc.out[seg][r0] = make_float2(psrc.get(seg, id), __int_as_float(id));
                }
                if (t2 < nn && r1 < K) {
                    const int id = order_key_index(c1);
                    sc.out[seg][r1] = make_float2(psrc.get(seg, id), __int_as_float(id));
                }
            }
            __syncwarp();
        }

        // Weights: gather the unbiased scores, renormalise, scale.
        float rowmax = 0.0f, denom_all = 1.0f;
        if constexpr (SCORE == kSoftmax) {
            float mx = m1;
#pragma unroll
            for (int o = L / 2; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, o));
            rowmax = mx;
            if (!a.renorm) {
                float s = 0.0f;
#pragma unroll
                for (int i = 0; i < C; ++i) s += softmax_num(key[i], rowmax, a.softcap);
#pragma unroll
                for (int o = L / 2; o >= 1; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
                denom_all = s;
            }
        }
        float w_loc[TPL];
        int id_loc[TPL];
        float sum = 0.0f;
#pragma unroll
        for (int q = 0; q < TPL; ++q) {
            const int t = sl + q * L;
            w_loc[q] = 0.0f;
            id_loc[q] = 0;
            if (t < K) {
                const float2 o = sc.out[seg][t];
                const float w = (SCORE == kSoftmax) ? softmax_num(o.x, rowmax, a.softcap) : o.x;
                w_loc[q] = w;
                id_loc[q] = __float_as_int(o.y);
                sum += w;
            }
        }
        float scale;
        if (a.renorm) {
#pragma unroll
            for (int o = L / 2; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFullMask, sum, o);
            scale = __fdividef(a.rsf, sum);
        } else {
            scale = (SCORE == kSoftmax) ? __fdividef(a.rsf, denom_all) : a.rsf;
        }
        if (valid) {
#pragma unroll
            for (int q = 0; q < TPL; ++q) {
                const int t = sl + q * L;
                if (t < K) {
                    a.weights[row * K + t] = w_loc[q] * scale;
                    a.ids[row * K + t] = id_loc[q];
                }
            }
        }
        __syncwarp();
    }
};

template <typename TIn, int E, int C, int SCORE, bool BIAS>
__global__ void __launch_bounds__(kSegThreads) route_segment_kernel(RouteArgs a) {
    using Router = SegRouter<E, C, SCORE, BIAS>;
    constexpr int L = Router::L;
    constexpr int R = Router::R;
    constexpr int WARPS = kSegThreads / 32;

    __shared__ __align__(16) typename Router::Scratch s_scratch[WARPS];
    __shared__ __align__(16) float s_p[WARPS][R * L * Router::CS];
    __shared__ __align__(16) float s_bias[BIAS ? Router::BIAS_FLOATS : 4];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int seg = lane / L;
    const int e0 = (lane % L) * C;

    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    if constexpr (BIAS) {
        Router::load_bias_padded(a.bias, s_bias, a.bias_bf16);
        __syncthreads();
    }

    const TIn* logits = static_cast<const TIn*>(a.logits);
    const int64_t step = (int64_t)gridDim.x * WARPS * R;
    for (int64_t row0 = ((int64_t)blockIdx.x * WARPS + warp) * R; row0 < a.M; row0 += step) {
        const int64_t row = row0 + seg;
        const bool valid = row < a.M;
        float x[C];
        if (valid) {
            ChunkLoader<TIn, C>::load(logits + row * E + e0, x);
        } else {
#pragma unroll
            for (int i = 0; i < C; ++i) x[i] = 0.0f;
        }
        Router::route(x, valid, row, s_bias, s_scratch[warp], a,
                      typename Router::StoredScores{s_p[warp]});
    }
}

// ---------------------------------------------------------------------------
// One thread per row, E <= 32.
// ---------------------------------------------------------------------------
template <typename TIn, int E, int SCORE, bool BIAS>
__global__ void __launch_bounds__(256) route_small_kernel(RouteArgs a) {
    const TIn* logits = static_cast<const TIn*>(a.logits);
    const int G = a.G, TG = a.TG, K = a.K;
    const int S = E / G;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; row < a.M; row += stride) {
        float x[E];
        ChunkLoader<TIn, E>::load(logits + row * E, x);
        float p[E], key[E];
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            p[i] = (SCORE == kSigmoid) ? sigmoid_f32(x[i]) : x[i];
            key[i] = BIAS ? p[i] + bias_as_used(__ldg(a.bias + i), a.bias_bf16) : p[i];
            mx = fmaxf(mx, x[i]);
        }
        // admissible experts: those of the TG best groups
        unsigned adm = (E >= 32) ? kFullMask : ((1u << E) - 1u);
        if (TG < G) {
            float gs[E];
#pragma unroll
            for (int h = 0; h < E; ++h) gs[h] = -INFINITY;
            for (int h = 0; h < G; ++h) {
                float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
                for (int i = 0; i < E; ++i)
                    if (i / S == h) top2_push(t1, t2, key[i]);
                gs[h] = (a.group_kind == kGroupTop2Sum) ? t1 + t2 : t1;
            }
            unsigned gmask = 0u;
            for (int h = 0; h < G; ++h) {
                int rank = 0;
                for (int o = 0; o < G; ++o) rank += beats(gs[o], o, gs[h], h) ? 1 : 0;
                if (rank < TG) gmask |= 1u << h;
            }
            adm = 0u;
#pragma unroll
            for (int i = 0; i < E; ++i)
                if ((gmask >> (i / S)) & 1u) adm |= 1u << i;
        }
        float denom_all = 1.0f;
        if (SCORE == kSoftmax && !a.renorm) {
            float s = 0.0f;
#pragma unroll
            for (int i = 0; i < E; ++i) s += softmax_num(x[i], mx, a.softcap);
            denom_all = s;
        }
        float sum = 0.0f;
        unsigned taken = 0u;
        for (int j = 0; j < K; ++j) {
            int bi = -1;
            float bv = -INFINITY, bp = 0.0f;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                if (((adm & ~taken) >> i) & 1u) {
                    if (bi < 0 || key[i] > bv) {
                        bv = key[i];
                        bi = i;
                        bp = p[i];
                    }
                }
            }
            if (bi < 0) bi = 0;  // unreachable for valid arguments
            taken |= 1u << bi;
            const float w = (SCORE == kSoftmax) ? softmax_num(bp, mx, a.softcap) : bp;
            sum += w;
            a.weights[row * K + j] = w;
            a.ids[row * K + j] = bi;
        }
        const float scale = a.renorm ? a.rsf / sum : ((SCORE == kSoftmax) ? a.rsf / denom_all : a.rsf);
        for (int j = 0; j < K; ++j) a.weights[row * K + j] *= scale;
    }
}

// ---------------------------------------------------------------------------
// One warp per row, any E <= 1024, any group shape, scalar loads.
// Dynamic shared memory per warp: 2*E floats + G floats + E bytes, 16-aligned.
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int generic_smem_per_warp(int E, int G) {
    return ((2 * E + G) * 4 + E + 15) / 16 * 16;
}

template <typename TIn, int SCORE>
__global__ void __launch_bounds__(128) route_generic_kernel(RouteArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int E = a.E, G = a.G, TG = a.TG, K = a.K;
    const int S = E / G;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int warps = blockDim.x >> 5;
    unsigned char* wbase = smem + (size_t)warp * generic_smem_per_warp(E, G);
    float* s_p = reinterpret_cast<float*>(wbase);
    float* s_key = s_p + E;
    float* s_gs = s_key + E;
    unsigned char* s_flag = reinterpret_cast<unsigned char*>(s_gs + G);  // bit0 kept, bit1 taken
    const TIn* logits = static_cast<const TIn*>(a.logits);

    for (int64_t row = (int64_t)blockIdx.x * warps + warp; row < a.M; row += (int64_t)gridDim.x * warps) {
        float mx = -INFINITY;
        for (int e = lane; e < E; e += 32) {
            const float x = load_scalar<TIn>(logits + row * E + e);
            const float p = (SCORE == kSigmoid) ? sigmoid_f32(x) : x;
            s_p[e] = p;
            s_key[e] = (a.bias != nullptr) ? p + bias_as_used(__ldg(a.bias + e), a.bias_bf16) : p;
            mx = fmaxf(mx, x);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, o));
        __syncwarp();
        for (int h = lane; h < G; h += 32) {
            float t1 = -INFINITY, t2 = -INFINITY;
            for (int j = 0; j < S; ++j) top2_push(t1, t2, s_key[h * S + j]);
            s_gs[h] = (a.group_kind == kGroupTop2Sum && S > 1) ? t1 + t2 : t1;
        }
        __syncwarp();
        for (int h = lane; h < G; h += 32) {
            int rank = 0;
            for (int o = 0; o < G; ++o) rank += beats(s_gs[o], o, s_gs[h], h) ? 1 : 0;
            const unsigned char kept = (TG >= G || rank < TG) ? 1 : 0;
            for (int j = 0; j < S; ++j) s_flag[h * S + j] = kept;
        }
        __syncwarp();
        float denom_all = 1.0f;
        if (SCORE == kSoftmax && !a.renorm) {
            float s = 0.0f;
            for (int e = lane; e < E; e += 32) s += softmax_num(s_p[e], mx, a.softcap);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
            denom_all = s;
        }
        float sum = 0.0f, my_w = 0.0f;
        int my_id = 0;
        for (int j = 0; j < K; ++j) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int e = lane; e < E; e += 32)
                if (s_flag[e] == 1 && (bi == 0x7fffffff || beats(s_key[e], e, bv, bi))) {
                    bv = s_key[e];
                    bi = e;
                }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(kFullMask, bv, o);
                const int oi = __shfl_xor_sync(kFullMask, bi, o);
                if ((oi != 0x7fffffff && bi == 0x7fffffff) || (oi != 0x7fffffff && beats(ov, oi, bv, bi))) {
                    bv = ov;
                    bi = oi;
                }
            }
            if (bi == 0x7fffffff) bi = 0;  // unreachable for valid arguments
            const float w = (SCORE == kSoftmax) ? softmax_num(s_p[bi], mx, a.softcap) : s_p[bi];
            sum += w;
            if (lane == j) {
                my_w = w;
                my_id = bi;
            }
            __syncwarp();
            if (lane == 0) s_flag[bi] = 3;
            __syncwarp();
        }
        const float scale = a.renorm ? a.rsf / sum : ((SCORE == kSoftmax) ? a.rsf / denom_all : a.rsf);
        if (lane < K) {
            a.weights[row * K + lane] = my_w * scale;
            a.ids[row * K + lane] = my_id;
        }
        __syncwarp();
    }
}

}  // namespace moe
