// Warp-per-row routing kernel for decode-sized batches: the SGLang MoE
// routing page's §2-§4 routing ("[SGLang] MoE 라우팅: 토큰에서 전문가로의 배분
// 알고리즘": softmax top-k, grouped top-k, sigmoid + correction_bias with the
// top-2-sum group score), shaped for the shortest dependency chain per row.
//
// One warp routes one token row at a time; lane l holds the C = E / 32
// consecutive experts [l C, (l + 1) C) in registers, read with one or two
// 16-byte loads (bf16 E = 256: one; fp32 E = 256: two) or C scalar loads, and
// its C bias values, loaded once per warp.
//
//  * Keys.  Selection key of each expert: sigmoid(x) + b (sigmoid with
//    correction bias), sigmoid(x) (sigmoid with group selection), x itself
//    (softmax, and sigmoid without bias or groups: both scores increase with
//    x).  Keys become order-preserving 32-bit integers (order_u32).
//  * Groups.  With G groups (G dividing 32) a group is 32 / G adjacent lanes:
//    their top-2 pairs meet through xor-shuffles, every lane ranks its group
//    against the G group scores (shuffles from each group's first lane, ties
//    to the lower group index), and lanes of dropped groups zero their keys
//    (zero is below every admissible key).
//  * Threshold.  tau = about the k-th largest of the 32 lane maxima, by k
//    rounds of __reduce_max_sync on the maxima made unique by the lane index
//    in their 5 low bits (each round's winner drops out); the maxima are
//    distinct experts, so every expert of the top k has a key >= tau; those
//    keys (about k + 4 on the benchmark workloads) are the candidates.
//  * Rank.  The candidates go to a per-warp list in lane order (positions
//    from a ballot prefix of the counts); lane t ranks candidate t by
//    counting the larger keys (16-byte broadcast reads) and writes it to
//    output slot `rank` if rank < k.  Equal keys, detected from the rank sum,
//    are ranked again with the lower expert index first.  A row with more
//    than 32 candidates takes k rounds of warp arg-max instead.
//  * Weights.  Lanes 0 .. k-1 read the slots, sum the scores for the
//    renormalisation with xor-shuffles and store weights and ids, k
//    consecutive words per row.
#pragma once

#include "routing_common.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kWarpRowWarps = 4;
constexpr int kWarpRowThreads = kWarpRowWarps * 32;

// The C logits of lane `lane` of a row as fp32: 16-byte loads when a lane's
// segment is a whole number of 16-byte vectors (the caller guarantees the
// alignment), else scalar loads.
template <typename TIn, int C>
__device__ __forceinline__ void warp_row_load(const TIn* rowp, int lane, float (&x)[C]) {
    constexpr int SEGB = C * (int)sizeof(TIn);
    const TIn* seg = rowp + lane * C;
    if constexpr (SEGB % 16 == 0) {
        const uint4* v = reinterpret_cast<const uint4*>(seg);
#pragma unroll
        for (int q = 0; q < SEGB / 16; ++q) {
            const uint4 u = __ldg(v + q);
            if constexpr (sizeof(TIn) == 2) {
                x[8 * q + 0] = bf16_lo(u.x); x[8 * q + 1] = bf16_hi(u.x);
                x[8 * q + 2] = bf16_lo(u.y); x[8 * q + 3] = bf16_hi(u.y);
                x[8 * q + 4] = bf16_lo(u.z); x[8 * q + 5] = bf16_hi(u.z);
                x[8 * q + 6] = bf16_lo(u.w); x[8 * q + 7] = bf16_hi(u.w);
            } else {
                x[4 * q + 0] = __uint_as_float(u.x); x[4 * q + 1] = __uint_as_float(u.y);
                x[4 * q + 2] = __uint_as_float(u.z); x[4 * q + 3] = __uint_as_float(u.w);
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if constexpr (sizeof(TIn) == 2)
                x[c] = __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(seg + c)))
                                       << 16);
            else
                x[c] = __ldg(reinterpret_cast<const float*>(seg + c));
        }
    }
}

// Per-warp scratch of warp_route_row: the candidate list and the output
// slots.
struct WarpRowScratch {
    float2 out[32];                 // by output slot: (score, id)
    __align__(16) uint32_t key[32]; // candidate list: orderable key
    int id[32];                     //   expert
    float p[32];                    //   unbiased score (softmax: logit)
};

// Route one token row with the whole warp: lane l holds the logits x and the
// bias values bl of experts [l C, (l + 1) C), C = E / 32.  Writes the row's
// k weights and ids (a.weights / a.ids, row `row`).  See route_warp_kernel.
template <int E, int SCORE, bool BIAS, bool GROUPED>
__device__ __forceinline__ void warp_route_row(const float (&x)[E / 32], const float (&bl)[E / 32], int64_t row,
                                               const RouteArgs& a, WarpRowScratch& sc) {
    constexpr int C = E / 32;
    constexpr bool KEYRAW = SCORE == kSoftmax || (!BIAS && !GROUPED);
    const int lane = threadIdx.x & 31;
    const int K = a.K;
    // ---- scores and selection keys
    float p[C], kf[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        p[c] = (SCORE == kSigmoid) ? sigmoid_f32(x[c]) : x[c];
        kf[c] = KEYRAW ? x[c] : (BIAS ? p[c] + bl[c] : p[c]);
    }
    uint32_t ku[C];
#pragma unroll
    for (int c = 0; c < C; ++c) ku[c] = order_u32(kf[c]);

    // ---- group selection
    if constexpr (GROUPED) {
        const int LPG = 32 / a.G;  // lanes per group
        float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
        for (int c = 0; c < C; ++c) top2_push(m1, m2, kf[c]);
        for (int o = 1; o < LPG; o <<= 1) {
            const float o1 = __shfl_xor_sync(kFullMask, m1, o);
            const float o2 = __shfl_xor_sync(kFullMask, m2, o);
            top2_merge(m1, m2, o1, o2);
        }
        const float gs = (a.group_kind == kGroupTop2Sum && E / a.G > 1) ? m1 + m2 : m1;
        const int g = lane / LPG;
        int rank = 0;
        for (int h = 0; h < a.G; ++h) {
            const float o = __shfl_sync(kFullMask, gs, h * LPG);
            rank += beats(o, h, gs, g) ? 1 : 0;
        }
        if (rank >= a.TG) {
#pragma unroll
            for (int c = 0; c < C; ++c) ku[c] = 0u;
        }
    }

    // ---- softmax normaliser over all experts (weights without renorm)
    float rowmax = 0.0f, denom_all = 1.0f;
    if constexpr (SCORE == kSoftmax) {
        rowmax = x[0];
#pragma unroll
        for (int c = 1; c < C; ++c) rowmax = fmaxf(rowmax, x[c]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) rowmax = fmaxf(rowmax, __shfl_xor_sync(kFullMask, rowmax, o));
        if (!a.renorm) {
            float s = 0.0f;
#pragma unroll
            for (int c = 0; c < C; ++c) s += softmax_num(x[c], rowmax, a.softcap);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o);
            denom_all = s;
        }
    }

    // ---- threshold: about the k-th largest of the 32 lane maxima.  Each
    // lane's maximum, its 5 low bits replaced by 31 - lane, is unique, so one
    // __reduce_max_sync per round finds the round's largest and its lane,
    // which drops out.  After k rounds, tau = that value with the 5 low bits
    // cleared: k distinct experts (the rounds' lane maxima) have keys >= tau,
    // so every expert of the top k has a key >= tau.
    uint32_t lm = ku[0];
#pragma unroll
    for (int c = 1; c < C; ++c) lm = max(lm, ku[c]);
    uint32_t tau = 0u;
    {
        uint32_t v = (lm & ~31u) | (31u - (uint32_t)lane);
#pragma unroll 1
        for (int j = 0; j < K; ++j) {
            tau = __reduce_max_sync(kFullMask, v);
            v = (v == tau) ? 0u : v;
        }
        tau &= ~31u;
    }
    // candidates: admissible keys >= tau
    uint32_t cm = 0u;
#pragma unroll
    for (int c = 0; c < C; ++c) cm |= (ku[c] >= tau && ku[c] != 0u) ? (1u << c) : 0u;
    const int cnt = __popc(cm);
    const int n = __reduce_add_sync(kFullMask, cnt);

    if (n >= K && n <= 32) {
        // ---- candidate list (key, id, score), in lane order
        const unsigned lt = (1u << lane) - 1u;
        int pos = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) pos += __popc(__ballot_sync(kFullMask, (cnt >> b) & 1) & lt) << b;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if ((cm >> c) & 1u) {
                sc.key[pos] = ku[c];
                sc.id[pos] = lane * C + c;
                sc.p[pos] = p[c];
                ++pos;
            }
        }
        const int jmax = (n + 3) & ~3;
        if (lane >= n && lane < jmax) sc.key[lane] = 0u;  // zero keys pad the list
        __syncwarp();
        // ---- rank of candidate `lane`: the candidates with larger keys
        uint32_t kt = 0u;
        int it = 0;
        float pt = 0.0f;
        if (lane < n) {
            kt = sc.key[lane];
            it = sc.id[lane];
            pt = sc.p[lane];
        }
        int rank = 0;
#pragma unroll
        for (int j4 = 0; j4 < 32; j4 += 4) {
            if (j4 < jmax) {
                const uint4 k4 = *reinterpret_cast<const uint4*>(&sc.key[j4]);
                rank += (k4.x > kt) + (k4.y > kt) + (k4.z > kt) + (k4.w > kt);
            }
        }
        // Distinct keys give the ranks 0 .. n-1; equal keys share a rank.
        // Then rank again, an equal key with a lower expert index first.
        const int rsum = __reduce_add_sync(kFullMask, lane < n ? rank : 0);
        if (rsum != n * (n - 1) / 2) {
            rank = 0;
            for (int j = 0; j < n; ++j) {
                const uint32_t kj = sc.key[j];
                rank += (kj > kt || (kj == kt && sc.id[j] < it)) ? 1 : 0;
            }
        }
        if (lane < n && rank < K) sc.out[rank] = make_float2(pt, __int_as_float(it));
    } else {
        // ---- rare rows (more than 32 candidates: massive ties, or too
        // few admissible lanes): k rounds of warp arg-max
#pragma unroll 1
        for (int j = 0; j < K; ++j) {
            uint32_t lb = ku[0];
#pragma unroll
            for (int c = 1; c < C; ++c) lb = max(lb, ku[c]);
            const uint32_t m = __reduce_max_sync(kFullMask, lb);
            const int w = __ffs(__ballot_sync(kFullMask, lb == m)) - 1;
            if (lane == w) {
                int ci = C - 1;
#pragma unroll
                for (int c = C - 2; c >= 0; --c) ci = (ku[c] == m) ? c : ci;
                float pw = p[0];
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    pw = (c == ci) ? p[c] : pw;
                    ku[c] = (c == ci) ? 0u : ku[c];
                }
                sc.out[j] = make_float2(pw, __int_as_float(lane * C + ci));
            }
        }
    }
    __syncwarp();  // the output slots are written before they are read

    // ---- weights: gather, renormalise, scale, store
    float wv = 0.0f;
    int iv = 0;
    if (lane < K) {
        const float2 o = sc.out[lane];
        wv = (SCORE == kSoftmax) ? softmax_num(o.x, rowmax, a.softcap) : o.x;
        iv = __float_as_int(o.y);
    }
    float wsum = wv;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) wsum += __shfl_xor_sync(kFullMask, wsum, o);
    float scale;
    if (a.renorm)
        scale = __fdividef(a.rsf, wsum);
    else
        scale = (SCORE == kSoftmax) ? __fdividef(a.rsf, denom_all) : a.rsf;
    if (lane < K) {
        a.weights[row * K + lane] = wv * scale;
        a.ids[row * K + lane] = iv;
    }
    __syncwarp();  // the slots are rewritten by the next row
}

// GROUPED: a.G > 1 with a.TG < a.G (some groups dropped).
// PARTS: the logits are the sum of a.nparts fp32 partials (TIn = float),
// added in a fixed order by the 4 warps of a block (one row per block, the
// grid covering the batch); a.logits_out, if set, receives the sums.
template <typename TIn, int E, int SCORE, bool BIAS, bool GROUPED, bool PARTS = false>
__global__ void __launch_bounds__(kWarpRowThreads) route_warp_kernel(RouteArgs a) {
    constexpr int C = E / 32;
    static_assert(E % 32 == 0 && C >= 1 && C <= 8, "warp-per-row shape");
    __shared__ WarpRowScratch s_scr[kWarpRowWarps];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * kWarpRowWarps;

    // The fused router's decode routing (PARTS) lets its dependent, the next
    // projection launch, set up at once: those CTAs take a whole SM each and
    // do not share SMs with this kernel's small blocks.
    if constexpr (PARTS) ptx::griddep_launch_dependents();
    // Inputs may be written by the previous kernel in the stream: wait for it.
    ptx::griddep_wait();

    float bl[C];
#pragma unroll
    for (int c = 0; c < C; ++c) bl[c] = BIAS ? bias_as_used(__ldg(a.bias + lane * C + c), a.bias_bf16) : 0.0f;

    const TIn* logits = static_cast<const TIn*>(a.logits);
    // PARTS: one row per block; the block's warps share the partial sums.
    const int64_t row0 = PARTS ? (int64_t)blockIdx.x : (int64_t)blockIdx.x * kWarpRowWarps + warp;
    const int64_t rstep = PARTS ? (int64_t)gridDim.x : nwarps;
    for (int64_t row = row0; row < a.M; row += rstep) {
        float x[C];
        if constexpr (PARTS) {
            static_assert(sizeof(TIn) == 4 && C % 4 == 0, "fp32 partials in 16-byte vectors");
            // Warp w adds the partials [w q, (w + 1) q) in order, then the
            // warps' sums are added in warp order (a fixed order).
            __shared__ __align__(16) float s_sum[kWarpRowWarps][E];
            const float* src = reinterpret_cast<const float*>(logits) + row * E + lane * C;
            const int q = (a.nparts + kWarpRowWarps - 1) / kWarpRowWarps;
            const int s0 = warp * q, s1 = min(a.nparts, s0 + q);
#pragma unroll
            for (int c = 0; c < C; ++c) x[c] = 0.0f;
#pragma unroll 8
            for (int s = s0; s < s1; ++s) {
#pragma unroll
                for (int v4 = 0; v4 < C / 4; ++v4) {
                    const float4 v = __ldcg(reinterpret_cast<const float4*>(src + s * a.part_stride) + v4);
                    x[4 * v4] += v.x;
                    x[4 * v4 + 1] += v.y;
                    x[4 * v4 + 2] += v.z;
                    x[4 * v4 + 3] += v.w;
                }
            }
#pragma unroll
            for (int v4 = 0; v4 < C / 4; ++v4)
                reinterpret_cast<float4*>(&s_sum[warp][lane * C])[v4] =
                    make_float4(x[4 * v4], x[4 * v4 + 1], x[4 * v4 + 2], x[4 * v4 + 3]);
            __syncthreads();
            if (warp != 0) break;  // one row per block: warp 0 routes it
#pragma unroll
            for (int c = 0; c < C; ++c) {
                float t = s_sum[0][lane * C + c];
#pragma unroll
                for (int w = 1; w < kWarpRowWarps; ++w) t += s_sum[w][lane * C + c];
                x[c] = t;
            }
            if (a.logits_out != nullptr) {
#pragma unroll
                for (int q = 0; q < C / 4; ++q)
                    reinterpret_cast<float4*>(a.logits_out + row * E + lane * C)[q] =
                        make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            }
        } else {
            warp_row_load<TIn, C>(logits + row * E, lane, x);
        }

        warp_route_row<E, SCORE, BIAS, GROUPED>(x, bl, row, a, s_scr[warp]);
    }
    // Let the next kernel in the stream launch only now: its blocks, waiting
    // on griddepcontrol.wait, would otherwise share this kernel's SMs (small
    // blocks co-reside) and take issue slots from it.
    if constexpr (!PARTS) ptx::griddep_launch_dependents();
}

}  // namespace moe
