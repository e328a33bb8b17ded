// Fused router: logits = hidden_states x router_weight on the tcgen05 tensor
// cores, then the biased grouped top-k routing on the fp32 accumulator
// (SGLang MoE routing page, §5 Fused MoE Router: the router projection and the
// top-k selection in one kernel, logits never stored; §4 for the routing).
//
// Design (one 128-token tile per cluster of SPLIT CTAs, one CTA per SM):
//   warp 0      TMA producer: A = hidden tile (128 x 64, K-major) and B = the
//               router weight tile (64 x 256) into a 4-stage ring, 128-byte
//               swizzle; B is K-major for (E, K) weights and MN-major for
//               (K, E) weights.
//   warp 1      allocates 256 TMEM columns and issues tcgen05.mma
//               (kind::f16, M=128, N=256, K=16, bf16 in, fp32 accumulate)
//               from one lane; tcgen05.commit frees a stage when its MMAs
//               are done and signals the epilogue after the last one.
//   warps 2..17 epilogue: the split-K partial sums are exchanged through
//               distributed shared memory (each CTA of the cluster owns
//               128/SPLIT rows and receives the other CTAs' partials for
//               them), summed in a fixed rank order, staged in shared memory
//               and routed by the same SegRouter body as the segment routing
//               kernel (8 lanes per row, 4 rows per warp in one pass).
// The K dimension is split across the SPLIT CTAs of a cluster so that enough
// SMs stream the hidden states (M=8192: 64 tiles x 2 = 128 CTAs).  A single
// tile with a long K (decode batches, M <= 128) takes fused_decode.cu
// instead.  Every barrier wait is bounded.
#include <cstdio>
#include <mutex>
#include <type_traits>
#include <unordered_map>

#include "fused_router.cuh"
#include "moe_routing.h"
#include "routing_kernels.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 16;                // four per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kFinStride = 8 * 36 + 4;  // floats per staged row: 8 chunks of 36 (bank spread)
constexpr uint64_t kWaitNs = 2000000000ull;

using Router = SegRouter<256, 32, kSigmoid, true>;
using RouterNB = SegRouter<256, 32, kSigmoid, false>;

static __device__ unsigned int g_watchdog_trips_fused;

struct FusedArgs {
    RouteArgs route;    // M, E, G, TG, K (topk), group_kind, renorm, rsf, bias, outputs
    float* logits_out;  // (M, 256) fp32 or nullptr
    int num_kb;         // K / 64
    int kb_per_split;   // k-blocks per CTA
};

// One 128-row tile with at least this many k-blocks takes the decode path
// (fused_decode.cu): K split over CTAs, partial logits in the workspace.
constexpr int kDecodeMinKb = 16;

// Bytes at the start of shared memory used first as the stage ring, then (after
// the main loop) as the split-K exchange and routing area.  With SPLIT = 2 that
// area holds this CTA's own rows (padded staged layout), the partner's partials
// (compact, received by one bulk copy) and the rows this CTA sends.
// Rows of the send/receive buffers are padded to an odd number of 16-byte
// chunks, so the 32 lanes of a warp (32 different rows) hit distinct banks.
constexpr int kPairStride = kBN + 4;
constexpr size_t kPairExchangeBytes =
    (size_t)(kBM / 2) * kFinStride * 4 + 2 * (size_t)(kBM / 2) * kPairStride * 4;
constexpr size_t kOverlayBytes = (size_t)kStages * kStageBytes > kPairExchangeBytes
                                     ? (size_t)kStages * kStageBytes
                                     : kPairExchangeBytes;

__host__ __device__ constexpr size_t fused_smem_bytes() {
    return 1024 + kOverlayBytes + Router::BIAS_FLOATS * 4 + 256;
}

// Owner-side staged logits row: chunk c (32 floats) at c * 36.
__device__ __forceinline__ int fin_off(int r, int col) { return r * kFinStride + (col >> 5) * 36 + (col & 31); }

template <int SPLIT>
struct FinScores {
    const float* fin;
    int warp_row0;
    __device__ __forceinline__ void store(int, float, float, float, float) const {}
    __device__ __forceinline__ float get(int seg, int e) const {
        const int r = warp_row0 + seg;  // rows past the owned range are padding
        return r < kBM / SPLIT ? sigmoid_f32(fin[fin_off(r, e)]) : 0.0f;
    }
};

template <int SPLIT, bool B_MN_MAJOR, bool BIAS>
__global__ void __launch_bounds__(kThreads, 1)
    fused_router_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        FusedArgs fa) {
    using R_t = typename std::conditional<BIAS, Router, RouterNB>::type;
    constexpr int ROWS = kBM / SPLIT;  // rows of the tile this CTA routes

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::smem_align<1024>(smem_raw);
    float* s_bias = reinterpret_cast<float*>(smem + kOverlayBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(s_bias + Router::BIAS_FLOATS);
    uint64_t* empty = full + kStages;
    uint64_t* accum = empty + kStages;
    uint64_t* recv_bar = accum + 1;  // SPLIT = 2: the partner's partials have landed
    uint64_t* sent_bar = accum + 2;  // SPLIT = 2: the partner holds our partials
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum + 3);
    volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* s_peer_abort = s_abort + 1;
    // Overlays of the stage ring, valid once the main loop is over: one slot
    // of partial sums per source CTA for the rows this CTA owns, in the
    // chunked staged-row layout; slot 0 is summed in place and then holds
    // the logits that are routed.
    float* slots = reinterpret_cast<float*>(smem);                                // [SPLIT][ROWS][292]
    float* fin = slots;
    // Router scratch reuses slots 1.. (and the rest of the ring) once they
    // have been summed into slot 0.
    auto* scratch = reinterpret_cast<typename R_t::Scratch*>(slots + (size_t)ROWS * kFinStride);
    static_assert((size_t)ROWS * kFinStride * 4 + kEpiWarps * sizeof(typename R_t::Scratch) <= kOverlayBytes,
                  "router scratch must fit in the stage ring");
    static_assert(SPLIT != 2 || kPairExchangeBytes <= kOverlayBytes, "pair exchange area");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const int m_tile = (int)(blockIdx.x / SPLIT);
    const int kb0 = (int)rank * fa.kb_per_split;
    int nkb = fa.num_kb - kb0;
    if (nkb > fa.kb_per_split) nkb = fa.kb_per_split;
    if (nkb < 0) nkb = 0;

    ptx::griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(accum, 1);
        ptx::mbar_init(recv_bar, 1);
        ptx::mbar_init(sent_bar, 1);
        *s_abort = 0;
        *s_peer_abort = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, 256);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();  // barriers initialised, TMEM address published
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // Everything above overlaps the previous kernel; inputs are read after it.
    // The producer starts streaming at once; the epilogue warps load the bias
    // meanwhile (their own barrier: they are the only readers).
    ptx::griddep_wait();
    if (warp >= 2) {
        if constexpr (BIAS) {
            for (int e = threadIdx.x - 64; e < 256; e += kEpiWarps * 32)
                s_bias[(e / 32) * Router::CS + e % 32] = __ldg(fa.route.bias + e);
        }
        ptx::named_barrier_sync(2, kEpiWarps * 32);
    }

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0 && nkb > 0) {
            const uint64_t pol_a = ptx::l2_policy_evict_first();
            const uint64_t pol_b = ptx::l2_policy_evict_last();
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % kStages;
                if (!ptx::mbar_wait(&empty[s], ((kb / kStages) & 1) ^ 1, kWaitNs)) {
                    *s_abort = 1;
                    atomicAdd(&g_watchdog_trips_fused, 1u);
                    break;
                }
                uint8_t* a_s = smem + (size_t)s * kStageBytes;
                uint8_t* b_s = a_s + kABytes;
                const int kc = (kb0 + kb) * kBK;
                ptx::mbar_arrive_expect_tx(&full[s], kStageBytes);
                ptx::tma_load_2d(a_s, &tmA, kc, m_tile * kBM, &full[s], pol_a);
                if constexpr (B_MN_MAJOR) {
#pragma unroll
                    for (int j = 0; j < kBN / 64; ++j)
                        ptx::tma_load_2d(b_s + j * 8192, &tmB, j * 64, kc, &full[s], pol_b);
                } else {
                    ptx::tma_load_2d(b_s, &tmB, kc, 0, &full[s], pol_b);
                }
            }
            // Leave only once the copies issued have landed (bounded).
            for (int k = 0; k < kStages && k < kb; ++k) {
                const int j = kb - 1 - k;
                ptx::mbar_wait(&full[j % kStages], (j / kStages) & 1, kWaitNs);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, kBN, B_MN_MAJOR);
            for (int kb = 0; kb < nkb && !*s_abort; ++kb) {
                const int s = kb % kStages;
                if (!ptx::mbar_wait(&full[s], (kb / kStages) & 1, kWaitNs)) {
                    *s_abort = 1;
                    atomicAdd(&g_watchdog_trips_fused, 1u);
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t a_addr = ptx::smem_u32(smem + (size_t)s * kStageBytes);
                const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t adesc = ptx::sdesc_sw128(a_addr + kk * 32, 16, 1024);
                    const uint64_t bdesc = B_MN_MAJOR ? ptx::sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                                      : ptx::sdesc_sw128(b_addr + kk * 32, 16, 1024);
                    ptx::umma_bf16(tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                }
                ptx::umma_commit(&empty[s]);
            }
            ptx::umma_commit(accum);
        }
    } else {
        // ---------------------------------------------------------- epilogue: wait for the accumulator
        if (!ptx::mbar_wait(accum, 0, kWaitNs)) {
            if (lane == 0) atomicAdd(&g_watchdog_trips_fused, 1u);
            *s_abort = 1;
        }
        ptx::tc_fence_after();
    }
    __syncwarp();

    // All MMAs of this CTA are complete (the epilogue waited on `accum`), so
    // the stage ring can be reused as the receive buffer.
    ptx::cluster_sync();

    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int r = q * 32 + lane;            // tile row of this thread's TMEM lane
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const bool epi = warp >= 2;
    const bool has_acc = nkb > 0;           // uniform over the CTA
    float* const recv = slots + (size_t)ROWS * kFinStride;  // SPLIT = 2: partner's partials [ROWS][260]
    float* const send = recv + (size_t)ROWS * kPairStride;  // SPLIT = 2: rows the partner owns [ROWS][260]
    if constexpr (SPLIT == 2) {
        // Own rows go to the staged layout, the partner's rows to a compact
        // send buffer that one bulk copy moves into the partner's receive
        // area (16-byte stores across the cluster are far slower).
        if (epi) {
            const int owner = r / ROWS;
            const int lr = r - owner * ROWS;
            const int part = (warp - 2) >> 2;
            const int c0 = part * 2;  // two 32-column chunks per warp
            const bool live = (int64_t)m_tile * kBM + r < fa.route.M;
            float v[64];
            __syncwarp();
            if (has_acc) {
                ptx::tmem_ld64(t_row + c0 * 32, v);
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] = 0.0f;
            }
            if (live) {
                if (owner == (int)rank) {
                    float* row = slots + (size_t)lr * kFinStride;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        *reinterpret_cast<float4*>(row + (c0 + i / 8) * 36 + 4 * (i % 8)) =
                            make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                } else {
                    float* row = send + (size_t)lr * kPairStride + c0 * 32;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        *reinterpret_cast<float4*>(row + 4 * i) =
                            make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::named_barrier_sync(3, kEpiWarps * 32);
            const uint32_t peer = rank ^ 1u;
            if (threadIdx.x == 64) {
                constexpr uint32_t kBytes = ROWS * kPairStride * 4;
                ptx::mbar_arrive_expect_tx(recv_bar, kBytes);
                const uint32_t dst = ptx::map_to_rank(ptx::smem_u32(recv), peer);
                const uint32_t mb = ptx::map_to_rank(ptx::smem_u32(recv_bar), peer);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    ptx::bulk_copy_to_cluster(dst + i * (kBytes / 4), ptx::smem_u32(send) + i * (kBytes / 4),
                                              kBytes / 4, mb);
            }
            if (!ptx::mbar_wait(recv_bar, 0, kWaitNs)) {
                if (threadIdx.x == 64) atomicAdd(&g_watchdog_trips_fused, 1u);
                *s_abort = 1;
            }
            // the partner's partials are here: its send buffer may be reused
            if (threadIdx.x == 64) ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_u32(sent_bar), peer));
        }
    } else if (epi) {
        // Every tile row's partial sums go to slot `rank` of the CTA that
        // owns the row (this CTA included).  tcgen05.ld is warp-collective:
        // whole warps load, lanes only choose the destination.
        const int owner = r / ROWS;
        float* own_row = slots + ((size_t)rank * ROWS + (r - owner * ROWS)) * kFinStride;
        const uint32_t dst = ptx::map_to_rank(ptx::smem_u32(own_row), owner);
        constexpr int PARTS = kEpiWarps / 4;           // warps per TMEM lane quarter
        constexpr int CPP = (kBN / 32) / PARTS;        // 32-column chunks per warp
        static_assert(CPP == 2, "one 64-column TMEM load per epilogue warp");
        const int part = (warp - 2) >> 2;
        const bool live = (int64_t)m_tile * kBM + r < fa.route.M;  // rows past M carry nothing
        const int c0 = part * CPP;
        float v[64];
        __syncwarp();
        if (has_acc) {
            ptx::tmem_ld64(t_row + c0 * 32, v);
        } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) v[i] = 0.0f;
        }
        if (live) {
            if (owner == (int)rank) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    *reinterpret_cast<float4*>(own_row + (c0 + i / 8) * 36 + 4 * (i % 8)) =
                        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    ptx::st_cluster_f32x4(dst + ((c0 + i / 8) * 36 + 4 * (i % 8)) * 4, v[4 * i], v[4 * i + 1],
                                          v[4 * i + 2], v[4 * i + 3]);
            }
        }
        if (*s_abort && part == 0)
            ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_u32(const_cast<int*>(s_peer_abort)), owner), 1u);
    }
    if constexpr (SPLIT != 2) ptx::cluster_sync();

    // Sum the SPLIT partials of the owned rows in rank order, all 128
    // epilogue threads in parallel, in place into slot 0.
    const int64_t row_base = (int64_t)m_tile * kBM + (int64_t)rank * ROWS;
    if (epi) {
        constexpr int COLS = kBN * ROWS / (kEpiWarps * 32);  // columns per thread
        const int t = threadIdx.x - 64;
        const int lr = t % ROWS;
        const int col0 = (t / ROWS) * COLS;
        const int64_t grow = row_base + lr;
#pragma unroll 1
        for (int col = col0; col < col0 + COLS; col += 4) {
            const int off = lr * kFinStride + (col >> 5) * 36 + (col & 31);
            if (grow >= fa.route.M) {
                *reinterpret_cast<float4*>(slots + off) = make_float4(0.f, 0.f, 0.f, 0.f);
                continue;
            }
            float4 acc = *reinterpret_cast<const float4*>(slots + off);
            if constexpr (SPLIT == 2) {
                // two partials: the sum is the same in either order
                const float4 v = *reinterpret_cast<const float4*>(recv + (size_t)lr * kPairStride + col);
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            } else {
                for (int src = 1; src < SPLIT; ++src) {
                    const float4 v =
                        *reinterpret_cast<const float4*>(slots + (size_t)src * ROWS * kFinStride + off);
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
            }
            *reinterpret_cast<float4*>(slots + off) = acc;
            if (fa.logits_out != nullptr && grow < fa.route.M)
                *reinterpret_cast<float4*>(fa.logits_out + grow * kBN + col) = acc;
        }
    }
    if constexpr (SPLIT == 2) {
        // The router scratch overlays the send buffer: wait until the partner
        // confirms our partials arrived.
        if (epi && !ptx::mbar_wait_cluster(sent_bar, 0, kWaitNs)) {
            if (threadIdx.x == 64) atomicAdd(&g_watchdog_trips_fused, 1u);
            *s_abort = 1;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 256);
    }

    // Routing of the owned rows by the epilogue warps (4 rows each per pass).
    if (epi) {
        const bool aborted = *s_abort || *s_peer_abort;
        const int ew = warp - 2;
        const int seg = lane / R_t::L;
        const int e0 = (lane % R_t::L) * 32;
        for (int base = 0; base < ROWS; base += kEpiWarps * R_t::R) {
            const int warp_row0 = base + ew * R_t::R;
            const int lr = warp_row0 + seg;
            const int64_t grow = row_base + lr;
            const bool valid = lr < ROWS && grow < fa.route.M;
            float x[32];
            if (lr < ROWS) {
                const float4* p = reinterpret_cast<const float4*>(fin + fin_off(lr, e0));
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 t = p[i];
                    x[4 * i] = t.x;
                    x[4 * i + 1] = t.y;
                    x[4 * i + 2] = t.z;
                    x[4 * i + 3] = t.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = 0.0f;
            }
            R_t::route(x, valid, grow, s_bias, scratch[ew], fa.route, FinScores<SPLIT>{fin, warp_row0});
            if (aborted && valid && (lane % R_t::L) == 0) {
                for (int t = 0; t < fa.route.K; ++t) fa.route.ids[grow * fa.route.K + t] = -1;
            }
        }
    }
}

template <int SPLIT, bool B_MN, bool BIAS>
int launch_fused(const CUtensorMap& tmA, const CUtensorMap& tmB, const FusedArgs& fa, int m_tiles,
                 cudaStream_t stream) {
    auto kern = fused_router_kernel<SPLIT, B_MN, BIAS>;
    {
        static std::mutex mu;
        static std::unordered_map<int, bool> done;  // device ordinal -> attributes set
        int dev = 0;
        cudaError_t gerr = cudaGetDevice(&dev);
        if (gerr != cudaSuccess) return set_cuda_error(gerr, "cudaGetDevice");
        std::lock_guard<std::mutex> lk(mu);
        if (!done[dev]) {
            cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)fused_smem_bytes());
            if (err != cudaSuccess) return set_cuda_error(err, "cudaFuncSetAttribute(fused router smem)");
            if (SPLIT > 8) {
                err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
                if (err != cudaSuccess) return set_cuda_error(err, "cudaFuncSetAttribute(cluster size)");
            }
            done[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(m_tiles * SPLIT), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = fused_smem_bytes();
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = SPLIT;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, fa);
    if (err != cudaSuccess) return set_cuda_error(err, "fused router launch");
    return MOE_OK;
}

template <bool B_MN, bool BIAS>
int launch_split(int split, const CUtensorMap& tmA, const CUtensorMap& tmB, const FusedArgs& fa,
                 int m_tiles, cudaStream_t st) {
    switch (split) {
        case 2: return launch_fused<2, B_MN, BIAS>(tmA, tmB, fa, m_tiles, st);
        case 4: return launch_fused<4, B_MN, BIAS>(tmA, tmB, fa, m_tiles, st);
        case 8: return launch_fused<8, B_MN, BIAS>(tmA, tmB, fa, m_tiles, st);
        default: return launch_fused<16, B_MN, BIAS>(tmA, tmB, fa, m_tiles, st);
    }
}

// Largest split whose cluster of one-CTA-per-SM blocks can be scheduled.
int max_schedulable_split(int dev) {
    static std::mutex mu;
    static std::unordered_map<int, int> cached;  // device ordinal -> split
    std::lock_guard<std::mutex> lk(mu);
    auto hit = cached.find(dev);
    if (hit != cached.end()) return hit->second;
    int best = 8;
    auto kern = fused_router_kernel<16, false, true>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fused_smem_bytes()) ==
            cudaSuccess &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = fused_smem_bytes();
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) best = 16;
    }
    cudaGetLastError();
    cached[dev] = best;
    return best;
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for moe_fused_router_topk_noalloc: a fixed device array that every
// GPU loading this library holds until the process exits.  Host code must not
// use the symbol itself as a pointer (on the host it only names the
// variable); its device address is looked up per device.
constexpr size_t kNoAllocScratchBytes = 2u << 20;  // 2 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up on
// the first call per device.
int noalloc_scratch(void** ptr) {
    static std::mutex mu;
    static std::unordered_map<int, void*> addr;  // device ordinal -> address of the array
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return set_cuda_error(err, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(mu);
    auto hit = addr.find(dev);
    if (hit == addr.end()) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (err != cudaSuccess) return set_cuda_error(err, "cudaGetSymbolAddress(no-alloc scratch)");
        hit = addr.emplace(dev, p).first;
    }
    *ptr = hit->second;
    return MOE_OK;
}

int read_fused_watchdog(unsigned int* count) {
    unsigned int v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_watchdog_trips_fused, sizeof(v));
    if (err != cudaSuccess) return set_cuda_error(err, "cudaMemcpyFromSymbol(fused watchdog)");
    *count = v;
    return MOE_OK;
}

}  // namespace moe

extern "C" {

size_t moe_fused_router_workspace_size(int64_t M, int32_t K, int32_t E) {
    if (M < 0 || K < 1 || E < 1) return (size_t)-1;
    // A single 128-token tile with a long K spreads K over several clusters
    // whose partial sums meet in the workspace; larger batches need none.
    if (M >= 1 && M <= moe::kBM && E == 256 && K % 64 == 0 && K / 64 >= moe::kDecodeMinKb)
        return moe::fused_decode_workspace_bytes(M, K / 64);
    return 0;
}

int moe_fused_router_topk(const void* hidden_states, const void* router_weight, int weight_layout,
                          const float* correction_bias, int64_t M, int32_t K, int32_t E,
                          int32_t topk, int32_t renormalize, int32_t num_expert_group,
                          int32_t topk_group, float routed_scaling_factor, float* topk_weights,
                          int32_t* topk_ids, float* logits_out, void* workspace,
                          size_t workspace_bytes, void* stream) {
    using namespace moe;
    const char* who = "moe_fused_router_topk";
    char msg[256];
    if (M < 0) {
        snprintf(msg, sizeof msg, "%s: M=%lld < 0", who, (long long)M);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (K < 1 || E < 1) {
        snprintf(msg, sizeof msg, "%s: K=%d and E=%d must be positive", who, K, E);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (weight_layout != MOE_WEIGHT_K_BY_E && weight_layout != MOE_WEIGHT_E_BY_K) {
        snprintf(msg, sizeof msg, "%s: weight_layout %d is not MOE_WEIGHT_K_BY_E or MOE_WEIGHT_E_BY_K", who,
                 weight_layout);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (num_expert_group < 1 || E % num_expert_group != 0 || topk_group < 1 || topk_group > num_expert_group ||
        topk < 1 || topk > topk_group * (E / num_expert_group) || !(routed_scaling_factor == routed_scaling_factor) ||
        routed_scaling_factor > 3.4e38f || routed_scaling_factor < -3.4e38f) {
        snprintf(msg, sizeof msg, "%s: invalid routing arguments (E=%d G=%d TG=%d topk=%d)", who, E,
                 num_expert_group, topk_group, topk);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (E != 256) {
        snprintf(msg, sizeof msg, "%s: E=%d; the fused router is built for E=256", who, E);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (K % 64 != 0) {
        snprintf(msg, sizeof msg, "%s: K=%d is not a multiple of 64", who, K);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (8 % num_expert_group != 0 || topk > 32) {
        snprintf(msg, sizeof msg, "%s: num_expert_group=%d / topk=%d not supported", who, num_expert_group, topk);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (M >= ((int64_t)1 << 31)) {  // tile counts and the outputs' row index stay within int32 grids
        snprintf(msg, sizeof msg, "%s: M=%lld >= 2^31", who, (long long)M);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (M == 0) return MOE_OK;
    if (!hidden_states || !router_weight || !topk_weights || !topk_ids)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fused_router_topk: null pointer argument");
    auto al = [](const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; };
    if (!al(hidden_states, 16) || !al(router_weight, 16) || (logits_out && !al(logits_out, 16)) ||
        !al(topk_weights, 4) || !al(topk_ids, 4) || (correction_bias && !al(correction_bias, 4)))
        return set_error(MOE_ERR_INVALID_ARG,
                         "moe_fused_router_topk: hidden_states/router_weight/logits_out must be 16-byte "
                         "aligned, outputs and bias 4-byte aligned");

    int dev = 0, sms = 0;
    int rc = sm_count(&dev, &sms);
    if (rc != MOE_OK) return rc;

    CUtensorMap tmA, tmB;
    cudaError_t err = encode_tmap_2d(&tmA, hidden_states, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)M,
                                     (uint64_t)K, (uint64_t)K * 2, kBK, kBM, true);
    if (err != cudaSuccess) return set_cuda_error(err, "cuTensorMapEncodeTiled(hidden_states)");
    const bool b_mn = weight_layout == MOE_WEIGHT_K_BY_E;
    if (b_mn)
        err = encode_tmap_2d(&tmB, router_weight, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)E,
                             (uint64_t)E * 2, 64, kBK, true);
    else
        err = encode_tmap_2d(&tmB, router_weight, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)E, (uint64_t)K,
                             (uint64_t)K * 2, kBK, kBN, true);
    if (err != cudaSuccess) return set_cuda_error(err, "cuTensorMapEncodeTiled(router_weight)");

    const int m_tiles = (int)((M + kBM - 1) / kBM);
    const int num_kb = K / kBK;
    const size_t ws_need = moe_fused_router_workspace_size(M, K, E);
    if (ws_need > 0 && (workspace == nullptr || workspace_bytes < ws_need ||
                        (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)) {
        snprintf(msg, sizeof msg, "%s: needs a 256-byte aligned workspace of %zu bytes (got %zu)", who, ws_need,
                 workspace_bytes);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    int split = 2;
    const int per = sms / (m_tiles > 0 ? m_tiles : 1);
    if (per >= 16) split = 16;
    else if (per >= 8) split = 8;
    else if (per >= 4) split = 4;
    if (split == 16 && max_schedulable_split(dev) < 16) split = 8;
    while (split > 2 && split > num_kb) split >>= 1;

    FusedArgs fa;
    fa.route.logits = nullptr;
    fa.route.bias = correction_bias;
    fa.route.M = M;
    fa.route.E = E;
    fa.route.G = num_expert_group;
    fa.route.TG = topk_group;
    fa.route.K = topk;
    fa.route.group_kind = kGroupTop2Sum;
    fa.route.renorm = renormalize ? 1 : 0;
    fa.route.rsf = routed_scaling_factor;
    fa.route.weights = topk_weights;
    fa.route.ids = topk_ids;
    fa.logits_out = logits_out;
    fa.num_kb = num_kb;
    fa.kb_per_split = (num_kb + split - 1) / split;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (ws_need > 0) {
        // one tile with a long K: split K over CTAs whose partial logits meet
        // in the workspace, then route them (two launches)
        return launch_fused_decode(tmA, router_weight, b_mn, fa.route, logits_out, num_kb, workspace, st);
    }
    if (b_mn)
        return correction_bias ? launch_split<true, true>(split, tmA, tmB, fa, m_tiles, st)
                               : launch_split<true, false>(split, tmA, tmB, fa, m_tiles, st);
    return correction_bias ? launch_split<false, true>(split, tmA, tmB, fa, m_tiles, st)
                           : launch_split<false, false>(split, tmA, tmB, fa, m_tiles, st);
}

int moe_fused_router_topk_noalloc(const void* hidden_states, const void* router_weight, int weight_layout,
                                  const float* correction_bias, int64_t M, int32_t K, int32_t E,
                                  int32_t topk, int32_t renormalize, int32_t num_expert_group,
                                  int32_t topk_group, float routed_scaling_factor, float* topk_weights,
                                  int32_t* topk_ids, float* logits_out, void* stream) {
    using namespace moe;
    const size_t need = moe_fused_router_workspace_size(M, K, E);
    if (need == (size_t)-1)
        return set_error(MOE_ERR_INVALID_ARG, "moe_fused_router_topk_noalloc: invalid sizes");
    if (need > kNoAllocScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "moe_fused_router_topk_noalloc: M=%lld, K=%d need %zu bytes of scratch; the built-in "
                 "scratch holds %zu (use moe_fused_router_topk with a workspace)",
                 (long long)M, K, need, kNoAllocScratchBytes);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    void* scratch = nullptr;
    if (need > 0) {
        int rc = noalloc_scratch(&scratch);
        if (rc != MOE_OK) return rc;
    }
    return moe_fused_router_topk(hidden_states, router_weight, weight_layout, correction_bias, M, K, E, topk,
                                 renormalize, num_expert_group, topk_group, routed_scaling_factor, topk_weights,
                                 topk_ids, logits_out, scratch, need, stream);
}

}  // extern "C"
