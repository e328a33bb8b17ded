// Two-phase streaming routing kernel for large batches with topk <= 8
// (E = 160 or 256): the SGLang MoE routing page's §2-§4 routing, split so
// that almost all per-row work runs one lane per row.
//
// A block is warp-specialised.  One TMA producer warp stages blocks of 32
// token rows into a shared-memory ring (2-D tensor map, 128-byte swizzle), as
// in route_staged_kernel.  Each staged block then goes through two phases:
//
//  * Phase 1 (a team of 8 warps, 8 lanes per row, C experts per lane): the
//    lane scores its C experts, takes its top-2, the row's kept groups and a
//    threshold tau that the k-th best admissible key is known to reach (the
//    k-th largest of the kept lanes' top-2 values, or with every group kept
//    of each lane's two largest 8-expert quarter maxima), and writes one bitmask
//    word per lane - its experts with key >= tau - band - to a per-block
//    table.  No compaction and no ranking here.  Two teams take alternate
//    blocks.
//  * Phase 2 (one of 8 dedicated warps, one lane per row): the lane walks its
//    row's candidate bits in ascending expert order, recomputes each
//    candidate's exact selection key from the staged logit and inserts it
//    into a sorted list of the 8 best.  Arrival in ascending index order plus
//    a strict comparison gives ties to the lower index, as the routing pages'
//    top-k does.  It then gathers the unbiased scores of the k winners,
//    renormalises, scales and stores, and releases the stage to the
//    producer.  Phase-2 warps never wait for phase 1 of later blocks, so the
//    latency of their candidate loops overlaps the streaming of the ring.
//
// Selection keys in phase 1 may be approximations of the phase-2 keys as long
// as |phase-1 key - phase-2 key| <= eps for every expert: then at least k
// experts have phase-2 keys >= tau - eps, so every phase-2 top-k expert has a
// phase-1 key >= tau - 2 eps and lies in the candidate set.  Two cases:
//  * sigmoid with every group kept (APPROX): key~ = 0.5 tanh(x/2) + (0.5 + b)
//    with the hardware tanh (one MUFU operation per expert instead of 1.5 and
//    no reciprocal); eps covers the tanh error bound kTanhApproxErr and the
//    fp32 roundings (scaled by the largest |bias|).
//  * sigmoid with group selection (exact phase 1): phase 1 uses the paired-
//    reciprocal sigmoid, phase 2 the single one; they differ by a few ulp, so
//    eps = 2^-20.
// Softmax keys are the raw logits in both phases (eps = 0).
#pragma once

#include "routing_staged.cuh"
#include "routing_threshold.cuh"

namespace moe {

constexpr int kStreamTeamWarps = 8;  // phase-1 warps per team (4 rows each)
constexpr int kStreamTeams = 2;      // phase-1 teams (alternate blocks)
constexpr int kStreamP2Warps = 8;    // phase-2 warps (block it goes to warp it mod 8)
constexpr int kStreamRows = 32;      // rows per stage (= lanes of a phase-2 warp)
constexpr int kStreamThreads = (1 + kStreamTeams * kStreamTeamWarps + kStreamP2Warps) * 32;
constexpr int kTabStride = 12;     // u32 words per row of the candidate table (48 B)
// Insert (v, e) into the descending list kk/ii.  Candidates arrive in
// ascending index order, so the strict comparison keeps equal keys in index
// order.
template <int N>
__device__ __forceinline__ void insert_desc(uint32_t (&kk)[N], int (&ii)[N], uint32_t v, int e) {
    bool c[N];
#pragma unroll
    for (int j = 0; j < N; ++j) c[j] = v > kk[j];
#pragma unroll
    for (int j = N - 1; j > 0; --j) {
        kk[j] = c[j - 1] ? kk[j - 1] : (c[j] ? v : kk[j]);
        ii[j] = c[j - 1] ? ii[j - 1] : (c[j] ? e : ii[j]);
    }
    kk[0] = c[0] ? v : kk[0];
    ii[0] = c[0] ? e : ii[0];
}

template <typename TIn, int E, int C, int SCORE, bool BIAS, bool APPROX>
struct StreamCfg {
    static constexpr int L = E / C;                      // lanes per row in phase 1
    static constexpr int R = 32 / L;                     // rows per warp in phase 1
    static constexpr int W = kStreamTeamWarps;
    static constexpr int RB = kStreamRows;
    static_assert(L == 8 && R * W == RB, "phase 1 covers the stage with 8 warps of 4 rows");
    static_assert(C <= 32 && C % 4 == 0, "one mask word per lane");
    static constexpr int ESZ = sizeof(TIn);
    static constexpr int CB = (E * ESZ + 127) / 128;     // 128-byte column blocks
    static constexpr int BOX_E = 128 / ESZ;
    static constexpr int STAGE_BYTES = CB * RB * 128;
    static constexpr int TAB_BYTES = RB * kTabStride * 4;
    static constexpr int CQ = (C / 4) | 1;               // padded lane-chunk layout (odd float4 count)
    static constexpr int CS = CQ * 4;
    static constexpr int VEC = (C * ESZ) % 16 == 0 ? 16 : 8;
    // Everything but the ring: alignment slack, phase-1 bias (or 0.5 + bias)
    // in the padded layout, phase-2 bias in expert order, scalars.
    static constexpr int FIXED = 1024 + L * CS * 4 + E * 4 + 64;
    // Stages: as many as fit in one block per SM (up to 12).
    static constexpr int S_FIT = (224 * 1024 - FIXED) / (STAGE_BYTES + TAB_BYTES + 24);
    static constexpr int S = S_FIT > 12 ? 12 : S_FIT;
    static_assert(S >= 4, "ring too shallow");
    static constexpr size_t SMEM = FIXED + (size_t)S * (STAGE_BYTES + TAB_BYTES + 24);
    static_assert(RB <= 256, "TMA box rows");
};

// Phase 2 of route_stream_kernel, run by phase-2 warp j (0 <= j < 8) for the
// blocks it = j, j + 8, ... of this CTA: one lane per staged row.
template <typename TIn, int E, int C, int SCORE, bool BIAS, bool APPROX>
__device__ __forceinline__ void route_stream_phase2(const RouteArgs& a, int64_t nblocks, int j,
                                                    const uint8_t* stages, uint32_t* tabs, const float* s_b2,
                                                    uint64_t* full, uint64_t* p1done, uint64_t* empty,
                                                    volatile int* s_abort) {
    using Cfg = StreamCfg<TIn, E, C, SCORE, BIAS, APPROX>;
    constexpr int RB = Cfg::RB, S = Cfg::S, P2 = kStreamP2Warps;
    const int lane = threadIdx.x & 31;
    const int K = a.K;
    int it = j;
    for (int64_t blk = blockIdx.x + (int64_t)j * gridDim.x; blk < nblocks; blk += (int64_t)P2 * gridDim.x, it += P2) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        // p1done: the team's masks are written; full (already complete): the
        // staged logits are visible to this warp.
        if (!ptx::mbar_wait(&p1done[s], ph, kWaitBudgetNs) || !ptx::mbar_wait(&full[s], ph, kWaitBudgetNs) ||
            *s_abort) {
            if (lane == 0 && !*s_abort) atomicAdd(&g_watchdog_trips_routing, 1u);
            *s_abort = 1;
            return;
        }
        const uint8_t* stage = stages + (size_t)s * Cfg::STAGE_BYTES;
        const int r = lane;
        const int64_t row = blk * RB + r;
        const bool valid = row < a.M;
        uint32_t* trow = tabs + (s * RB + r) * kTabStride;
        const uint4 w03 = *reinterpret_cast<const uint4*>(trow);
        const uint4 w47 = *reinterpret_cast<const uint4*>(trow + 4);
        const uint4 meta = *reinterpret_cast<const uint4*>(trow + 8);
        uint32_t wd[8] = {w03.x, w03.y, w03.z, w03.w, w47.x, w47.y, w47.z, w47.w};
        int n = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) n += __popc(wd[q]);
        if (valid && n < K) {
            // fewer candidates than K (NaN scores): take every expert of the
            // kept groups
            const uint32_t all = (C == 32) ? 0xffffffffu : ((1u << C) - 1u);
            n = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                wd[q] = ((meta.x >> q) & 1u) ? all : 0u;
                trow[q] = wd[q];
                n += __popc(wd[q]);
            }
        }
        if (!valid) n = 0;
        const int nmax = __reduce_max_sync(kFullMask, n);
        uint32_t occ = 0u;  // words with candidates left
#pragma unroll
        for (int q = 0; q < 8; ++q) occ |= (wd[q] != 0u ? 1u : 0u) << q;

        uint32_t kk[8];
        int ii[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            kk[q] = 0u;
            ii[q] = 0;
        }
        // Branch-free two-deep software pipeline: while candidate t is
        // inserted, candidate t + 1 is scored (its MUFU operations in flight)
        // and candidate t + 2 located and loaded.  Slots past the lane's own
        // count insert key 0, which changes nothing (every real key is >= 1).
        uint32_t cur = 0u;
        int wi = 0;
        auto next_cand = [&]() -> int {
            const bool sw = (cur == 0u);
            const int nw = max(__ffs(occ) - 1, 0);
            wi = sw ? nw : wi;
            occ = sw ? (occ & (occ - 1u)) : occ;
            const uint32_t fresh = trow[wi];
            cur = sw ? fresh : cur;
            const int b = max(__ffs(cur) - 1, 0);
            cur &= cur - 1u;
            return wi * C + b;
        };
        auto load_x = [&](int e) { return staged_scalar<TIn>(staged_addr<RB>(stage, r, e * Cfg::ESZ)); };
        auto score = [&](float xv, float bv) -> float {
            if constexpr (SCORE == kSigmoid) return BIAS ? sigmoid_f32(xv) + bv : sigmoid_f32(xv);
            return xv;
        };
        int e1 = next_cand();
        float x1 = load_x(e1), b1 = BIAS ? s_b2[e1] : 0.0f;
        int e2 = next_cand();
        float x2 = load_x(e2), b2 = BIAS ? s_b2[e2] : 0.0f;
        float k1 = score(x1, b1);
        for (int t = 0; t < nmax; ++t) {
            const float k2 = score(x2, b2);
            const int e3 = next_cand();
            const float x3 = load_x(e3), b3 = BIAS ? s_b2[e3] : 0.0f;
            insert_desc(kk, ii, (t < n) ? order_u32(k1) : 0u, e1);
            e1 = e2;
            k1 = k2;
            e2 = e3;
            x2 = x3;
            b2 = b3;
        }

        // weights of the K winners: unbiased scores, renormalised, scaled
        float xw[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            xw[q] = (q < K) ? staged_scalar<TIn>(staged_addr<RB>(stage, r, ii[q] * Cfg::ESZ)) : 0.0f;
        float rowmax = 0.0f;
        if constexpr (SCORE == kSoftmax) rowmax = a.renorm ? xw[0] : __uint_as_float(meta.y);
        float wv[8];
        float sum = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            wv[q] = 0.0f;
            if (q < K) {
                wv[q] = (SCORE == kSoftmax) ? softmax_num(xw[q], rowmax, a.softcap) : sigmoid_f32(xw[q]);
                sum += wv[q];
            }
        }
        float scale;
        if (a.renorm)
            scale = __fdividef(a.rsf, sum);
        else
            scale = (SCORE == kSoftmax) ? __fdividef(a.rsf, __uint_as_float(meta.z)) : a.rsf;
        // all lanes have read the stage and the table: release the stage
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[s]);
        if (valid) {
            float* wo = a.weights + row * K;
            int32_t* io = a.ids + row * K;
            if (K == 8 && ((reinterpret_cast<uintptr_t>(a.weights) | reinterpret_cast<uintptr_t>(a.ids)) & 15) == 0) {
                reinterpret_cast<float4*>(wo)[0] = make_float4(wv[0] * scale, wv[1] * scale, wv[2] * scale, wv[3] * scale);
                reinterpret_cast<float4*>(wo)[1] = make_float4(wv[4] * scale, wv[5] * scale, wv[6] * scale, wv[7] * scale);
                reinterpret_cast<int4*>(io)[0] = make_int4(ii[0], ii[1], ii[2], ii[3]);
                reinterpret_cast<int4*>(io)[1] = make_int4(ii[4], ii[5], ii[6], ii[7]);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (q < K) {
                        wo[q] = wv[q] * scale;
                        io[q] = ii[q];
                    }
                }
            }
        }
    }
}

template <typename TIn, int E, int C, int SCORE, bool BIAS, bool APPROX>
__global__ void __launch_bounds__(kStreamThreads, 1)
    route_stream_kernel(const __grid_constant__ CUtensorMap tmap, RouteArgs a, int64_t nblocks) {
    using Cfg = StreamCfg<TIn, E, C, SCORE, BIAS, APPROX>;
    constexpr int W = Cfg::W, R = Cfg::R, RB = Cfg::RB, S = Cfg::S, L = Cfg::L, CS = Cfg::CS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = ptx::smem_align<1024>(smem_raw);
    uint8_t* stages = base;
    uint32_t* tabs = reinterpret_cast<uint32_t*>(stages + (size_t)S * Cfg::STAGE_BYTES);
    float* s_b1 = reinterpret_cast<float*>(tabs + S * RB * kTabStride);  // phase 1: padded (0.5 +) bias
    float* s_b2 = s_b1 + L * CS;                                          // phase 2: bias by expert
    uint64_t* full = reinterpret_cast<uint64_t*>(s_b2 + E);
    uint64_t* p1done = full + S;
    uint64_t* empty = p1done + S;
    volatile int* s_abort = reinterpret_cast<volatile int*>(empty + S);
    float* s_band = reinterpret_cast<float*>(empty + S) + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    ptx::griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&p1done[s], W);
            ptx::mbar_init(&empty[s], 1);
        }
        *s_abort = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tmap);
    }
    // Bias tables and the candidate band (built by one consumer warp).
    auto build_tables = [&]() {
        float bmax = 0.0f;
        for (int e = lane; e < E; e += 32) {
            const float b = BIAS ? bias_as_used(__ldg(a.bias + e), a.bias_bf16) : 0.0f;
            s_b2[e] = b;
            s_b1[(e / C) * CS + e % C] = APPROX ? 0.5f + b : b;
            bmax = fmaxf(bmax, fabsf(b));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFullMask, bmax, o));
        if (lane == 0) {
            float band = 0.0f;
            if constexpr (SCORE == kSigmoid) {
                // eps = tanh term + fp32 roundings of keys of size up to 2 + |b|
                // (APPROX), or the pair/single sigmoid difference; band = 2 eps.
                const float round = (bmax + 2.0f) * (1.0f / 2097152.0f);  // 4 ulp at 2 + |b|
                band = APPROX ? 2.0f * (0.5f * kTanhApproxErr + round) : 2.0f * (kPairKeyErr + round);
            }
            *s_band = band;
        }
    };
    __syncthreads();  // barriers initialised
    ptx::griddep_wait();

    constexpr int NT = kStreamTeams, P2 = kStreamP2Warps;
    // Warp roles: 0 producer, 1..P2 phase 2, then the phase-1 teams.
    if (warp == 0) {
        // ---------------- producer: one elected lane issues the TMA loads
        if (lane == 0) {
            const uint64_t policy = ptx::l2_policy_evict_first();
            int it = 0;
            for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x, ++it) {
                const int s = it % S;
                if (!ptx::mbar_wait(&empty[s], ((it / S) & 1) ^ 1, kWaitBudgetNs) || *s_abort) {
                    *s_abort = 1;
                    atomicAdd(&g_watchdog_trips_routing, 1u);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&full[s], Cfg::STAGE_BYTES);
                uint8_t* dst = stages + (size_t)s * Cfg::STAGE_BYTES;
#pragma unroll
                for (int cb = 0; cb < Cfg::CB; ++cb)
                    ptx::tma_load_2d(dst + cb * (RB * 128), &tmap, cb * Cfg::BOX_E, (int)(blk * RB), &full[s],
                                     policy);
            }
            for (int k = 0; k < S && k < it; ++k) {
                const int j = it - 1 - k;
                ptx::mbar_wait(&full[j % S], (j / S) & 1, kWaitBudgetNs);
            }
        }
        return;
    }

    // The producer streams from the start; the consumer warps build the bias
    // tables meanwhile.
    if (warp == 1) build_tables();
    ptx::named_barrier_sync(1, (NT * W + P2) * 32);
    if (warp <= P2) {
        route_stream_phase2<TIn, E, C, SCORE, BIAS, APPROX>(a, nblocks, warp - 1, stages, tabs, s_b2,
                                                           full, p1done, empty, s_abort);
        return;
    }

    // -------------------- phase-1 teams
    const int team = (warp - 1 - P2) / W;
    const int tw = (warp - 1 - P2) % W;  // warp within the team
    const float band = *s_band;
    const int seg = lane / L;
    const int sl = lane % L;
    const int sbase = seg * L;
    const int e0 = sl * C;
    const int G = a.G, TG = a.TG, K = a.K;
    const int P = L / G;  // lanes per group (the dispatcher guarantees G | L)
    const int g = sl / P;
    const bool all_groups = (TG == G);
    const int nsel_lanes = all_groups ? L : TG * P;
    const int need = (K + 1) >> 1;
    const int r1 = tw * R + seg;  // phase-1 row of this lane within the stage

    int it = team;
    for (int64_t blk = blockIdx.x + (int64_t)team * gridDim.x; blk < nblocks;
         blk += (int64_t)NT * gridDim.x, it += NT) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!ptx::mbar_wait(&full[s], ph, kWaitBudgetNs) || *s_abort) {
            if (lane == 0 && !*s_abort) atomicAdd(&g_watchdog_trips_routing, 1u);
            *s_abort = 1;
            break;
        }
        const uint8_t* stage = stages + (size_t)s * Cfg::STAGE_BYTES;
        uint32_t* tab = tabs + s * RB * kTabStride;

        // ============ phase 1: keys, top-2, kept groups, threshold, mask word
        {
            const int64_t row = blk * RB + r1;
            const bool valid = row < a.M;
            float x[C];
            if constexpr (Cfg::VEC == 16) {
#pragma unroll
                for (int q = 0; q < C * Cfg::ESZ / 16; ++q) {
                    uint4 v = *reinterpret_cast<const uint4*>(staged_addr<RB>(stage, r1, e0 * Cfg::ESZ + 16 * q));
                    if constexpr (sizeof(TIn) == 2 && SCORE == kSigmoid && !APPROX) {
                        v.x = clamp_bf16x2_for_sigmoid(v.x);
                        v.y = clamp_bf16x2_for_sigmoid(v.y);
                        v.z = clamp_bf16x2_for_sigmoid(v.z);
                        v.w = clamp_bf16x2_for_sigmoid(v.w);
                    }
                    if constexpr (sizeof(TIn) == 2) {
                        x[8 * q + 0] = bf16_lo(v.x); x[8 * q + 1] = bf16_hi(v.x);
                        x[8 * q + 2] = bf16_lo(v.y); x[8 * q + 3] = bf16_hi(v.y);
                        x[8 * q + 4] = bf16_lo(v.z); x[8 * q + 5] = bf16_hi(v.z);
                        x[8 * q + 6] = bf16_lo(v.w); x[8 * q + 7] = bf16_hi(v.w);
                    } else {
                        x[4 * q + 0] = __uint_as_float(v.x); x[4 * q + 1] = __uint_as_float(v.y);
                        x[4 * q + 2] = __uint_as_float(v.z); x[4 * q + 3] = __uint_as_float(v.w);
                    }
                }
            } else {
#pragma unroll
                for (int q = 0; q < C * Cfg::ESZ / 8; ++q) {
                    uint2 v = *reinterpret_cast<const uint2*>(staged_addr<RB>(stage, r1, e0 * Cfg::ESZ + 8 * q));
                    if constexpr (sizeof(TIn) == 2 && SCORE == kSigmoid && !APPROX) {
                        v.x = clamp_bf16x2_for_sigmoid(v.x);
                        v.y = clamp_bf16x2_for_sigmoid(v.y);
                    }
                    if constexpr (sizeof(TIn) == 2) {
                        x[4 * q + 0] = bf16_lo(v.x); x[4 * q + 1] = bf16_hi(v.x);
                        x[4 * q + 2] = bf16_lo(v.y); x[4 * q + 3] = bf16_hi(v.y);
                    } else {
                        x[2 * q + 0] = __uint_as_float(v.x); x[2 * q + 1] = __uint_as_float(v.y);
                    }
                }
            }

            float key[C];
            const float* bl = s_b1 + sl * CS;
#pragma unroll
            for (int q = 0; q < C / 4; ++q) {
                const float4 b = reinterpret_cast<const float4*>(bl)[q];
                unsigned long long k01, k23;
                if constexpr (SCORE == kSigmoid && APPROX) {
                    const unsigned long long h01 = mul2(pack2(x[4 * q], x[4 * q + 1]), pack2(0.5f, 0.5f));
                    const unsigned long long h23 = mul2(pack2(x[4 * q + 2], x[4 * q + 3]), pack2(0.5f, 0.5f));
                    const unsigned long long t01 = pack2(tanh_approx(lo2(h01)), tanh_approx(hi2(h01)));
                    const unsigned long long t23 = pack2(tanh_approx(lo2(h23)), tanh_approx(hi2(h23)));
                    k01 = fma2(t01, pack2(0.5f, 0.5f), pack2(b.x, b.y));
                    k23 = fma2(t23, pack2(0.5f, 0.5f), pack2(b.z, b.w));
                } else if constexpr (SCORE == kSigmoid) {
                    float x0 = x[4 * q], x1 = x[4 * q + 1], x2 = x[4 * q + 2], x3 = x[4 * q + 3];
                    if constexpr (sizeof(TIn) != 2) {
                        x0 = fmaxf(x0, kSigmoidClamp);
                        x1 = fmaxf(x1, kSigmoidClamp);
                        x2 = fmaxf(x2, kSigmoidClamp);
                        x3 = fmaxf(x3, kSigmoidClamp);
                    }
                    k01 = sigmoid_pair(pack2(x0, x1));
                    k23 = sigmoid_pair(pack2(x2, x3));
                    if constexpr (BIAS) {
                        k01 = add2(k01, pack2(b.x, b.y));
                        k23 = add2(k23, pack2(b.z, b.w));
                    }
                } else {
                    k01 = pack2(x[4 * q], x[4 * q + 1]);
                    k23 = pack2(x[4 * q + 2], x[4 * q + 3]);
                }
                key[4 * q + 0] = lo2(k01);
                key[4 * q + 1] = hi2(k01);
                key[4 * q + 2] = lo2(k23);
                key[4 * q + 3] = hi2(k23);
            }
            float m1 = 0.0f, m2 = 0.0f;
            float tau = -INFINITY;
            const bool quarters = (C == 32) && all_groups;
            if (quarters) {
                // every group kept: the threshold comes from the maxima of the
                // lane's four 8-expert quarters (distinct experts)
                float q[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float* k8 = key + 8 * (u % (C / 8));
                    q[u] = fmax3(fmax3(k8[0], k8[1], k8[2]), fmax3(k8[3], k8[4], k8[5]), fmaxf(k8[6], k8[7]));
                }
                // the lane's two largest quarter maxima: the K-th largest of
                // the row's 16 is still a lower bound (distinct experts)
                const float ah = fmaxf(q[0], q[1]), al = fminf(q[0], q[1]);
                const float ch = fmaxf(q[2], q[3]), cl = fminf(q[2], q[3]);
                tau = row_kth2<L>(fmaxf(ah, ch), fmax3(fminf(ah, ch), al, cl), K, m1);  // m1: row max
            } else {
                top2_of(key, m1, m2);
            }

            // kept groups (exact keys here: APPROX is only used with every
            // group kept)
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
                    const float o = __shfl_sync(kFullMask, gs, sbase + h * P);
                    rank += (o > gs) || (o == gs && h < g);
                }
                gsel = rank < TG;
            }

            // threshold: the K-th best phase-1 key is >= tau
            if (quarters) {
            } else if (need > nsel_lanes) {
                tau = -INFINITY;
            } else if (need == nsel_lanes) {
                float v = gsel ? m2 : INFINITY;
#pragma unroll
                for (int o = L / 2; o >= 1; o >>= 1) v = fminf(v, __shfl_xor_sync(kFullMask, v, o));
                tau = v;
            } else {
                if constexpr (L == 8) {
                    float vmax;
                    tau = row_kth2<L>(gsel ? m1 : -INFINITY, gsel ? m2 : -INFINITY, K, vmax);
                } else {
                    float top[8];
                    segment_top8<L>(gsel ? m1 : -INFINITY, gsel ? m2 : -INFINITY, top);
                    tau = kth_of_sorted8(top, K);
                }
            }
            const float lo = tau - band;

            // bit i set iff key[i] >= lo, i.e. key[i] - lo >= +0: gather the
            // sign bits of the differences with integer multiply-adds
            uint32_t below = 0u;
            {
                const unsigned long long nlo = pack2(-lo, -lo);
#pragma unroll
                for (int i = 0; i < C; i += 2) {
                    const unsigned long long d = add2(pack2(key[i], key[i + 1]), nlo);
                    uint32_t s0, s1;
                    asm("mul.hi.u32 %0, %1, 2;" : "=r"(s0) : "r"((uint32_t)d));
                    asm("mul.hi.u32 %0, %1, 2;" : "=r"(s1) : "r"((uint32_t)(d >> 32)));
                    asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(below) : "r"(s0), "r"(1u << i));
                    asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(below) : "r"(s1), "r"(2u << i));
                }
            }
            const uint32_t cmask = (C == 32) ? 0xffffffffu : ((1u << C) - 1u);
            const uint32_t mask = (gsel && valid) ? (~below & cmask) : 0u;
            uint32_t* trow = tab + r1 * kTabStride;
            trow[sl] = mask;

            const unsigned keep = (__ballot_sync(kFullMask, gsel) >> sbase) & 0xffu;
            if constexpr (SCORE == kSoftmax) {
                // row max and (without renormalisation) the full softmax
                // denominator, for the phase-2 weights
                float mx = m1;
                if (!quarters) {
#pragma unroll
                    for (int o = L / 2; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, o));
                }
                float den = 1.0f;
                if (!a.renorm) {
                    float sacc = 0.0f;
#pragma unroll
                    for (int i = 0; i < C; ++i) sacc += softmax_num(x[i], mx, a.softcap);
#pragma unroll
                    for (int o = L / 2; o >= 1; o >>= 1) sacc += __shfl_xor_sync(kFullMask, sacc, o);
                    den = sacc;
                }
                if (sl == 0) {
                    trow[9] = __float_as_uint(mx);
                    trow[10] = __float_as_uint(den);
                }
            }
            if (sl == 0) trow[8] = keep;
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&p1done[s]);

    }
}

}  // namespace moe
