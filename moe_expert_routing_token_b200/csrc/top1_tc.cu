// Tensor-core top-1 router: the tensor-core branch of the fused router of the
// SGLang MoE routing page ("[SGLang] MoE 라우팅: 토큰에서 전문가로의 배분
// 알고리즘", §5 Fused MoE Router) for router weights stored (E, K), E up to
// 256.  Per token row:
//
//   l_e  = sum_k h[k] * W[e][k]          bf16 inputs, fp32 accumulation (TMEM)
//   id   = arg-max_e l_e                 lowest index among equal logits
//   w    = 1 / sum_e exp(cap(l_e) - cap(l_id)),   cap(x) = c * tanh(x / c)
//
// The arg-max is taken on the raw logits, as in the CUDA-core kernel: the cap
// is monotone, so the raw maximum is a maximum of the capped values too.
//
// Design (one 128-row tile per cluster of SPLIT CTAs, the K dimension split
// among them):
//   warp 0      TMA producer: the hidden tile (128 x 64, K-major) and the
//               weight tile (NP x 64, K-major; NP = E rounded up to 16, 32,
//               64, 128 or 256, rows past E zero-filled by the copy) into a
//               ring, 128-byte swizzle.
//   warp 1      allocates the TMEM accumulator and issues tcgen05.mma
//               (kind::f16, M = 128, N = NP, K = 16) from one lane;
//               tcgen05.commit frees a stage and signals the accumulator.
//   warps 2-5   epilogue, one TMEM lane (one tile row) per thread.  With
//               SPLIT = 1 the thread routes its row from TMEM.  Otherwise CTA
//               `rank` owns rows [rank * 128/SPLIT, (rank + 1) * 128/SPLIT)
//               of the tile: every CTA stores its partial logits of each row
//               into slot `rank` of the owner's shared memory
//               (st.shared::cluster), and the owner sums the slots in rank
//               order, SPLIT threads per row, each over every SPLIT-th
//               expert, the arg-max and the denominator meeting through
//               shuffles.
// The projection is 2 E flops per 2-byte hidden value, far below the tensor
// cores' ridge: the kernel streams the hidden states from HBM and the split
// along K lets small batches use more SMs.  Every barrier wait is bounded.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <mutex>
#include <type_traits>
#include <unordered_map>

#include "moe_routing.h"
#include "routing_common.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace moe {

int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);
int sm_count(int* dev, int* sms);

static __device__ unsigned int g_watchdog_trips_top1;

namespace {

constexpr int kTcBM = 128;
constexpr int kTcBK = 64;
constexpr int kTcThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr uint64_t kTcWaitNs = 2000000000ull;

template <int NP>
struct TcRing {
    static constexpr int A_BYTES = kTcBM * kTcBK * 2;
    static constexpr int B_BYTES = NP * kTcBK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int S = (192 * 1024 / STAGE) < 10 ? (192 * 1024 / STAGE) : 10;  // ring depth
    static constexpr int TCOLS = NP < 32 ? 32 : NP;  // TMEM columns: a power of two >= 32
    static constexpr int NP32 = (NP + 31) / 32 * 32;
    static_assert(NP % 16 == 0 && NP >= 16 && NP <= 256, "UMMA N for M = 128");
    static_assert(STAGE % 1024 == 0, "128-byte swizzled tiles start on 1024-byte boundaries");
    static_assert(S >= 2, "ring too shallow");
};

template <int NP, int SPLIT>
struct TcCfg : TcRing<NP> {
    using R = TcRing<NP>;
    static constexpr int ROWS = kTcBM / SPLIT;  // tile rows a CTA routes
    // floats per partial row: the SPLIT threads of a row read every SPLIT-th
    // column, so a stride of SPLIT (mod 32) puts a warp's reads in 32 banks
    static constexpr int PS = R::NP32 + SPLIT;
    static constexpr size_t SLOT_BYTES = SPLIT > 1 ? (size_t)SPLIT * ROWS * PS * 4 : 0;
    static constexpr size_t RING_BYTES = (size_t)R::S * R::STAGE;
    static constexpr size_t OVERLAY = RING_BYTES > SLOT_BYTES ? RING_BYTES : SLOT_BYTES;
    static constexpr size_t SMEM = 1024 + OVERLAY + 256;
    static_assert(SPLIT == 1 || SPLIT == 2 || SPLIT == 4 || SPLIT == 8 || SPLIT == 16, "split");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct TcArgs {
    int64_t M;
    int E;
    int num_kb;         // K / 64
    int kb_per_split;   // k-blocks per CTA of a cluster
    float softcap;
    float* weights;     // (M, 1)
    int32_t* ids;       // (M, 1)
    float* logits_out;  // (M, E) or nullptr
};

// 16 consecutive fp32 columns of this thread's TMEM lane, waited for.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Running arg-max in ascending expert order: a later expert replaces the
// current one only if strictly larger (ties keep the lower index).
__device__ __forceinline__ void argmax_step(float v, int e, bool& any, float& bv, int& best) {
    if (!any || v > bv) {
        bv = v;
        best = e;
        any = true;
    }
}

template <int NP, int SPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
    top1_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcArgs ta) {
    using Cfg = TcCfg<NP, SPLIT>;
    constexpr int S = Cfg::S;
    constexpr int ROWS = Cfg::ROWS;
    constexpr int PS = Cfg::PS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::smem_align<1024>(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::OVERLAY);
    uint64_t* empty = full + S;
    uint64_t* accum = empty + S;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);  // this CTA gave up
    volatile int* s_abort_in = s_abort + 1;  // a CTA of the cluster gave up (set remotely)
    float* slots = reinterpret_cast<float*>(smem);  // [SPLIT][ROWS][PS] after the main loop

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = SPLIT > 1 ? ptx::cluster_ctarank() : 0u;
    const int m_tile = (int)(blockIdx.x / SPLIT);
    const int kb0 = (int)rank * ta.kb_per_split;
    int nkb = ta.num_kb - kb0;
    if (nkb > ta.kb_per_split) nkb = ta.kb_per_split;
    if (nkb < 0) nkb = 0;
    const int E = ta.E;

    ptx::griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(accum, 1);
        *s_abort = 0;
        *s_abort_in = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, Cfg::TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // The inputs may be written by the previous kernel in the stream.
    ptx::griddep_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0 && nkb > 0) {
            const uint64_t pol_a = ptx::l2_policy_evict_first();
            const uint64_t pol_b = ptx::l2_policy_evict_last();
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % S;
                if (!ptx::mbar_wait(&empty[s], ((kb / S) & 1) ^ 1, kTcWaitNs)) {
                    *s_abort = 1;
                    atomicAdd(&g_watchdog_trips_top1, 1u);
                    break;
                }
                uint8_t* a_s = smem + (size_t)s * Cfg::STAGE;
                const int kc = (kb0 + kb) * kTcBK;
                ptx::mbar_arrive_expect_tx(&full[s], Cfg::STAGE);
                ptx::tma_load_2d(a_s, &tmA, kc, m_tile * kTcBM, &full[s], pol_a);
                ptx::tma_load_2d(a_s + Cfg::A_BYTES, &tmB, kc, 0, &full[s], pol_b);
            }
            // leave only once the copies issued have landed (bounded)
            for (int k = 0; k < S && k < kb; ++k) {
                const int j = kb - 1 - k;
                ptx::mbar_wait(&full[j % S], (j / S) & 1, kTcWaitNs);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && nkb > 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kTcBM, NP, false);
            for (int kb = 0; kb < nkb && !*s_abort; ++kb) {
                const int s = kb % S;
                if (!ptx::mbar_wait(&full[s], (kb / S) & 1, kTcWaitNs)) {
                    *s_abort = 1;
                    atomicAdd(&g_watchdog_trips_top1, 1u);
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t a_addr = ptx::smem_u32(smem + (size_t)s * Cfg::STAGE);
                const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < kTcBK / 16; ++kk) {
                    const uint64_t adesc = ptx::sdesc_sw128(a_addr + kk * 32, 16, 1024);
                    const uint64_t bdesc = ptx::sdesc_sw128(b_addr + kk * 32, 16, 1024);
                    ptx::umma_bf16(tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                }
                ptx::umma_commit(&empty[s]);
            }
            ptx::umma_commit(accum);
        }
    } else {
        // ---------------------------------------------------------- epilogue: accumulator ready
        if (nkb > 0 && !ptx::mbar_wait(accum, 0, kTcWaitNs)) {
            if (lane == 0) atomicAdd(&g_watchdog_trips_top1, 1u);
            *s_abort = 1;
        }
        ptx::tc_fence_after();
    }
    __syncwarp();

    const bool epi = warp >= 2;
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const bool have = nkb > 0;

    if constexpr (SPLIT == 1) {
        // ---- one thread per row, logits from TMEM
        if (epi) {
            const int r = q * 32 + lane;
            const int64_t row = (int64_t)m_tile * kTcBM + r;
            const bool live = row < ta.M;
            bool any = false;
            float bv = 0.0f;
            int best = 0;
#pragma unroll 1
            for (int c0 = 0; c0 < E; c0 += 16) {
                float v[16];
                __syncwarp();
                if (have) {
                    tmem_ld16(t_row + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (c0 + i < E) {
                        argmax_step(v[i], c0 + i, any, bv, best);
                        if (live && ta.logits_out) ta.logits_out[row * E + c0 + i] = v[i];
                    }
                }
            }
            float den = 0.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < E; c0 += 16) {
                float v[16];
                __syncwarp();
                if (have) {
                    tmem_ld16(t_row + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (c0 + i < E) den += softmax_num(v[i], bv, ta.softcap);
            }
            if (live) {
                ta.weights[row] = 1.0f / den;
                ta.ids[row] = *s_abort ? -1 : best;
            }
        }
    } else {
        // ---- partial logits to the row owners
        ptx::cluster_sync();  // every CTA's ring is idle: it becomes the slots
        // rows past the batch are neither sent nor routed
        const int r = q * 32 + lane;
        if (epi && __any_sync(kFullMask, (int64_t)m_tile * kTcBM + r < ta.M)) {
            const uint32_t owner = (uint32_t)(r / ROWS);
            const uint32_t dst =
                ptx::map_to_rank(ptx::smem_u32(slots + ((size_t)rank * ROWS + (r % ROWS)) * PS), owner);
#pragma unroll 1
            for (int c0 = 0; c0 < E; c0 += 16) {
                float v[16];
                __syncwarp();
                if (have) {
                    tmem_ld16(t_row + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
                }
                if constexpr (PS % 4 == 0) {
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        ptx::st_cluster_f32x4(dst + (c0 + i) * 4, v[i], v[i + 1], v[i + 2], v[i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) ptx::st_cluster_u32(dst + (c0 + i) * 4, __float_as_uint(v[i]));
                }
            }
            if (*s_abort)
                ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_u32((const void*)s_abort_in), owner), 1u);
        }
        ptx::cluster_sync();  // every slot written

        if (epi) {
            const int t = threadIdx.x - 64;
            const int rr = t / SPLIT;  // owned row
            const int j = t % SPLIT;   // this thread takes experts j, j + SPLIT, ...
            const int64_t row = (int64_t)m_tile * kTcBM + (int64_t)rank * ROWS + rr;
            const bool live = row < ta.M;
            float* const mine = slots + (size_t)rr * PS;
            bool any = false;
            float bv = 0.0f;
            int best = 0;
#pragma unroll 1
            for (int c = j; c < E; c += SPLIT) {
                float s = mine[c];
#pragma unroll
                for (int src = 1; src < SPLIT; ++src) s += slots[((size_t)src * ROWS + rr) * PS + c];
                mine[c] = s;
                argmax_step(s, c, any, bv, best);
                if (live && ta.logits_out) ta.logits_out[row * E + c] = s;
            }
            // arg-max over the row's SPLIT threads (adjacent lanes)
#pragma unroll
            for (int off = SPLIT / 2; off >= 1; off >>= 1) {
                const float ov = __shfl_xor_sync(kFullMask, bv, off);
                const int oi = __shfl_xor_sync(kFullMask, best, off);
                const bool oa = __shfl_xor_sync(kFullMask, any ? 1 : 0, off) != 0;
                if (oa && (!any || ov > bv || (ov == bv && oi < best))) {
                    bv = ov;
                    best = oi;
                    any = true;
                }
            }
            float den = 0.0f;
#pragma unroll 1
            for (int c = j; c < E; c += SPLIT) den += softmax_num(mine[c], bv, ta.softcap);
#pragma unroll
            for (int off = SPLIT / 2; off >= 1; off >>= 1) den += __shfl_xor_sync(kFullMask, den, off);
            if (live && j == 0) {
                ta.weights[row] = 1.0f / den;
                ta.ids[row] = (*s_abort || *s_abort_in) ? -1 : best;
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, Cfg::TCOLS);
    }
}

// Per device: shared-memory size set, and whether a cluster of SPLIT such
// blocks can be scheduled.
template <int NP, int SPLIT>
int prepare_tc(int dev, bool* schedulable) {
    static std::mutex mu;
    static std::unordered_map<int, bool> ok;  // device ordinal -> schedulable
    std::lock_guard<std::mutex> lk(mu);
    auto it = ok.find(dev);
    if (it != ok.end()) {
        *schedulable = it->second;
        return MOE_OK;
    }
    auto kern = top1_tc_kernel<NP, SPLIT>;
    constexpr size_t smem = TcCfg<NP, SPLIT>::SMEM;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return set_cuda_error(err, "cudaFuncSetAttribute(top-1 router smem)");
    bool can = true;
    if (SPLIT > 8) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return set_cuda_error(err, "cudaFuncSetAttribute(top-1 router cluster size)");
    }
    if (SPLIT > 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(SPLIT, 1, 1);
        cfg.blockDim = dim3(kTcThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = SPLIT;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        err = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
        if (err != cudaSuccess) {
            (void)cudaGetLastError();
            clusters = 0;
        }
        can = clusters > 0;
    }
    ok[dev] = can;
    *schedulable = can;
    return MOE_OK;
}

template <int NP, int SPLIT>
int launch_tc(const CUtensorMap& tmA, const CUtensorMap& tmB, const TcArgs& ta, int m_tiles, cudaStream_t st) {
    auto kern = top1_tc_kernel<NP, SPLIT>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(m_tiles * SPLIT), 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = TcCfg<NP, SPLIT>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (SPLIT > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = SPLIT;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, ta);
    if (err != cudaSuccess) return set_cuda_error(err, "top-1 router launch");
    return MOE_OK;
}

template <int NP>
int launch_np(int dev, int split, const CUtensorMap& tmA, const CUtensorMap& tmB, const TcArgs& ta, int m_tiles,
              cudaStream_t st) {
    bool can = false;
    int rc = MOE_OK;
    if (split >= 16) {
        rc = prepare_tc<NP, 16>(dev, &can);
        if (rc != MOE_OK) return rc;
        if (can) return launch_tc<NP, 16>(tmA, tmB, ta, m_tiles, st);
        split = 8;
    }
    if (split >= 8) {
        rc = prepare_tc<NP, 8>(dev, &can);
        if (rc != MOE_OK) return rc;
        if (can) return launch_tc<NP, 8>(tmA, tmB, ta, m_tiles, st);
        split = 4;
    }
    if (split >= 4) {
        rc = prepare_tc<NP, 4>(dev, &can);
        if (rc != MOE_OK) return rc;
        if (can) return launch_tc<NP, 4>(tmA, tmB, ta, m_tiles, st);
        split = 2;
    }
    if (split >= 2) {
        rc = prepare_tc<NP, 2>(dev, &can);
        if (rc != MOE_OK) return rc;
        if (can) return launch_tc<NP, 2>(tmA, tmB, ta, m_tiles, st);
    }
    rc = prepare_tc<NP, 1>(dev, &can);
    if (rc != MOE_OK) return rc;
    return launch_tc<NP, 1>(tmA, tmB, ta, m_tiles, st);
}

}  // namespace

// Split along K for a batch of m_tiles 128-row tiles over num_kb k-blocks:
// the largest of 1, 2, 4, 8, 16 that keeps the CTAs within the SMs and gives
// every CTA at least two k-blocks.  (The kernel's ta.kb_per_split is derived
// from the split the launch actually uses.)
int top1_tc_split(int64_t m_tiles, int num_kb, int sms) {
    int split = 1;
    while (split < 16 && m_tiles * split * 2 <= sms && split * 4 <= num_kb) split *= 2;
    return split;
}

// The tensor-core top-1 router for (E, K) weights, K a multiple of 64 and
// E <= 256 (sizes, pointers and alignment validated by the caller).
int launch_top1_tc(const void* h, const void* w, int64_t M, int K, int E, float softcap, float* weights,
                   int32_t* ids, float* logits_out, cudaStream_t st) {
    int dev = 0, sms = 0;
    int rc = sm_count(&dev, &sms);
    if (rc != MOE_OK) return rc;
    const int np = E <= 16 ? 16 : E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;
    const int64_t m_tiles = (M + kTcBM - 1) / kTcBM;
    if (m_tiles > (int64_t)(1 << 26))
        return set_error(MOE_ERR_UNSUPPORTED, "moe_fused_router_top1: M above the tensor-core kernel's grid");
    CUtensorMap tmA, tmB;
    cudaError_t err = encode_tmap_2d(&tmA, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)M, (uint64_t)K,
                                     (uint64_t)K * 2, kTcBK, kTcBM, true);
    if (err != cudaSuccess) return set_cuda_error(err, "cuTensorMapEncodeTiled(hidden_states)");
    err = encode_tmap_2d(&tmB, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)E, (uint64_t)K, (uint64_t)K * 2,
                         kTcBK, (uint32_t)np, true);
    if (err != cudaSuccess) return set_cuda_error(err, "cuTensorMapEncodeTiled(router_weight)");
    const int num_kb = K / kTcBK;
    const int split = top1_tc_split(m_tiles, num_kb, sms);
    TcArgs ta;
    ta.M = M;
    ta.E = E;
    ta.num_kb = num_kb;
    ta.softcap = softcap;
    ta.weights = weights;
    ta.ids = ids;
    ta.logits_out = logits_out;
    const int mt = (int)m_tiles;
    // The k-blocks per CTA follow the split that is launched: a cluster size
    // the device cannot schedule falls back to the next smaller one.
    auto go = [&](auto np_tag) -> int {
        constexpr int NP = decltype(np_tag)::value;
        int s = split;
        while (s > 1) {
            bool can = false;
            int r2 = MOE_OK;
            switch (s) {
                case 16: r2 = prepare_tc<NP, 16>(dev, &can); break;
                case 8: r2 = prepare_tc<NP, 8>(dev, &can); break;
                case 4: r2 = prepare_tc<NP, 4>(dev, &can); break;
                default: r2 = prepare_tc<NP, 2>(dev, &can); break;
            }
            if (r2 != MOE_OK) return r2;
            if (can) break;
            s >>= 1;
        }
        ta.kb_per_split = (num_kb + s - 1) / s;
        return launch_np<NP>(dev, s, tmA, tmB, ta, mt, st);
    };
    switch (np) {
        case 16: return go(std::integral_constant<int, 16>{});
        case 32: return go(std::integral_constant<int, 32>{});
        case 64: return go(std::integral_constant<int, 64>{});
        case 128: return go(std::integral_constant<int, 128>{});
        default: return go(std::integral_constant<int, 256>{});
    }
}

int read_top1_watchdog(unsigned int* count) {
    unsigned int v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_watchdog_trips_top1, sizeof(v));
    if (err != cudaSuccess) return set_cuda_error(err, "cudaMemcpyFromSymbol(top-1 watchdog)");
    *count = v;
    return MOE_OK;
}

}  // namespace moe
