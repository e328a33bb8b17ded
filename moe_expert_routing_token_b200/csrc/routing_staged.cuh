// Streaming routing kernel for large batches: a TMA producer warp stages
// blocks of RB token rows into a multi-stage shared-memory ring (2-D tensor
// map, 128-byte swizzle) while W consumer warps route the rows already
// staged.  The memory-level parallelism therefore no longer depends on how
// many consumer warps are resident: S stages of STAGE_BYTES per block are in
// flight regardless.  Consumers read their lane chunks from the swizzled
// stage (conflict-free 16-byte loads in natural element order) and recompute
// a candidate's unbiased score from the staged logit instead of keeping a
// per-warp score buffer.
//
// Routing semantics are those of SegRouter (routing_kernels.cuh).
#pragma once

#include "routing_kernels.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kStagedWarps = 8;             // consumer warps per block

// Incremented when a barrier wait times out (a kernel then stops early and
// leaves its outputs unspecified); read back by moe_watchdog_trips().
static __device__ unsigned int g_watchdog_trips_routing;

template <typename TIn, int E, int C, int SCORE, bool BIAS>
struct StagedCfg {
    using Router = SegRouter<E, C, SCORE, BIAS>;
    static constexpr int W = kStagedWarps;
    static constexpr int R = Router::R;
    static constexpr int RB = W * R;                      // rows per stage
    static constexpr int ESZ = sizeof(TIn);
    static constexpr int CB = (E * ESZ + 127) / 128;      // 128-byte column blocks
    static constexpr int BOX_E = 128 / ESZ;               // elements per box row
    static constexpr int STAGE_BYTES = CB * RB * 128;
    // Stages: as many as fit (up to 4) while two blocks share an SM
    // (<= ~113 KB each); a layout that cannot keep 2 stages that way runs
    // one block per SM with 4 stages.
    static constexpr int FIXED = 1024 + W * (int)sizeof(typename Router::Scratch) + Router::BIAS_FLOATS * 4 + 128;
    static constexpr int S2 = (113 * 1024 - FIXED) / STAGE_BYTES;
    static constexpr int S = S2 >= 2 ? (S2 > 4 ? 4 : S2) : 4;
    static constexpr int VEC = (C * ESZ) % 16 == 0 ? 16 : 8;  // bytes per chunk load
    static constexpr int BIAS_FLOATS = Router::BIAS_FLOATS;
    static constexpr size_t SMEM = 1024 + (size_t)S * STAGE_BYTES + W * sizeof(typename Router::Scratch) +
                                   BIAS_FLOATS * 4 + 2 * S * 8 + 16;
    static_assert(RB <= 256, "TMA box rows");
};

// Byte address of (row r, byte b of the row) inside a stage written by TMA
// with 128-byte swizzle: 16-byte chunk index XOR (r mod 8).
template <int RB>
__device__ __forceinline__ const uint8_t* staged_addr(const uint8_t* stage, int r, int b) {
    return stage + (b >> 7) * (RB * 128) + r * 128 + ((((b & 127) >> 4) ^ (r & 7)) << 4) + (b & 15);
}

template <typename TIn>
__device__ __forceinline__ float staged_scalar(const uint8_t* p);
template <>
__device__ __forceinline__ float staged_scalar<float>(const uint8_t* p) {
    return *reinterpret_cast<const float*>(p);
}
template <>
__device__ __forceinline__ float staged_scalar<__nv_bfloat16>(const uint8_t* p) {
    return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(p)) << 16);
}

template <typename TIn, int E, int C, int SCORE, bool BIAS>
struct StagedScores {
    using Cfg = StagedCfg<TIn, E, C, SCORE, BIAS>;
    const uint8_t* stage;
    int warp_row0;  // stage row of segment 0 of this warp
    __device__ __forceinline__ void store(int, float, float, float, float) const {}
    __device__ __forceinline__ float get(int seg, int e) const {
        const float x = staged_scalar<TIn>(staged_addr<Cfg::RB>(stage, warp_row0 + seg, e * Cfg::ESZ));
        return SCORE == kSigmoid ? sigmoid_f32(x) : x;
    }
};

template <typename TIn, int E, int C, int SCORE, bool BIAS>
__global__ void __launch_bounds__((kStagedWarps + 1) * 32)
    route_staged_kernel(const __grid_constant__ CUtensorMap tmap, RouteArgs a, int64_t nblocks) {
    using Cfg = StagedCfg<TIn, E, C, SCORE, BIAS>;
    using Router = typename Cfg::Router;
    constexpr int W = Cfg::W, R = Cfg::R, RB = Cfg::RB, S = Cfg::S, L = Router::L;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = ptx::smem_align<1024>(smem_raw);
    uint8_t* stages = base;
    auto* scratch = reinterpret_cast<typename Router::Scratch*>(stages + (size_t)S * Cfg::STAGE_BYTES);
    float* s_bias = reinterpret_cast<float*>(scratch + W);
    uint64_t* full = reinterpret_cast<uint64_t*>(s_bias + Cfg::BIAS_FLOATS);
    uint64_t* empty = full + S;
    volatile int* s_abort = reinterpret_cast<volatile int*>(empty + S);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    ptx::griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], W);
        }
        *s_abort = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tmap);
    }
    // Everything above overlaps the previous kernel in the stream; global
    // inputs are read only after it has finished.
    ptx::griddep_wait();
    if constexpr (BIAS) Router::load_bias_padded(a.bias, s_bias, a.bias_bf16);
    __syncthreads();

    if (warp == W) {
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
            // Do not leave while copies may still land: wait (bounded) for the
            // last stages issued.
            for (int k = 0; k < S && k < it; ++k) {
                const int j = it - 1 - k;
                ptx::mbar_wait(&full[j % S], (j / S) & 1, kWaitBudgetNs);
            }
        }
        return;
    }

    // -------------------- consumers
    const int seg = lane / L;
    const int e0 = (lane % L) * C;
    const int warp_row0 = warp * R;
    int it = 0;
    for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x, ++it) {
        const int s = it % S;
        if (!ptx::mbar_wait(&full[s], (it / S) & 1, kWaitBudgetNs) || *s_abort) {
            if (lane == 0 && !*s_abort) atomicAdd(&g_watchdog_trips_routing, 1u);
            *s_abort = 1;
            break;
        }
        const uint8_t* stage = stages + (size_t)s * Cfg::STAGE_BYTES;
        const int r = warp_row0 + seg;
        const int64_t row = blk * RB + r;
        const bool valid = row < a.M;

        float x[C];
        if constexpr (Cfg::VEC == 16) {
#pragma unroll
            for (int q = 0; q < C * Cfg::ESZ / 16; ++q) {
                uint4 v = *reinterpret_cast<const uint4*>(staged_addr<RB>(stage, r, e0 * Cfg::ESZ + 16 * q));
                if constexpr (sizeof(TIn) == 2 && SCORE == kSigmoid) {
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
                uint2 v = *reinterpret_cast<const uint2*>(staged_addr<RB>(stage, r, e0 * Cfg::ESZ + 8 * q));
                if constexpr (sizeof(TIn) == 2 && SCORE == kSigmoid) {
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
        Router::template route<sizeof(TIn) == 2>(x, valid, row, s_bias, scratch[warp], a,
                                                 StagedScores<TIn, E, C, SCORE, BIAS>{stage, warp_row0});
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[s]);
    }
}

}  // namespace moe
