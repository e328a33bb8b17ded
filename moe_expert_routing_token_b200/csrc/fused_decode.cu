// Fused router for decode-sized batches (one 128-token tile, M <= 128): the
// router projection of the SGLang MoE routing page (§5 Fused MoE Router)
// followed by its §4 biased grouped top-k, in two launches shaped for latency.
//
//  1. fused_decode_proj_kernel: the hidden size is cut into nsplit ranges of
//     k-blocks and the 256 experts into 4 slices of 64, one CTA per (range,
//     slice) (no clusters): each CTA does a quarter of the tensor work of a
//     full-width split, so 4x as many SMs share the projection.  Warp 0
//     streams the hidden tile (128 x 64, K-major) and the weight slice
//     (64 x 64, K-major for (E, K) weights, MN-major for (K, E)) with TMA into
//     a 4-stage ring; warp 1 issues tcgen05.mma (M = 128, N = 64, K = 16) into
//     64 TMEM columns; warps 2-5 read the accumulator rows of the batch (one
//     TMEM lane per thread) and store them, fp32, to the workspace as partial
//     logits [nsplit][M][256] (this slice's 64 columns).
//  2. route_warp_kernel with partial inputs (programmatic dependent launch):
//     one block per token row; its 4 warps each add a quarter of the nsplit
//     partials, the quarters are added in warp order (a fixed order, so the
//     result is deterministic), and warp 0 routes the row.
// The logits cross L2 once as partials (at most 2 MiB), instead of each
// split's partials meeting in one CTA: with a single tile, a cluster
// exchange or a last-CTA reduction puts the whole reduction on a few SMs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "fused_router.cuh"
#include "moe_routing.h"
#include "routing_warp.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace moe {

static __device__ unsigned int g_watchdog_trips_decode;

namespace {

constexpr int kDBM = 128;
constexpr int kDE = 256;     // experts (columns of a partial row)
constexpr int kDBN = 64;     // experts per CTA (N of the MMA)
constexpr int kDSlices = kDE / kDBN;
constexpr int kDBK = 64;
constexpr int kDStages = 4;
constexpr int kDABytes = kDBM * kDBK * 2;
constexpr int kDBBytes = kDBN * kDBK * 2;
constexpr int kDStageBytes = kDABytes + kDBBytes;
constexpr int kDThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr size_t kDSmem = 1024 + (size_t)kDStages * kDStageBytes + 256;
constexpr uint64_t kDWaitNs = 2000000000ull;
constexpr int kDecodeKbPerCta = 4;            // target k-blocks per CTA
constexpr size_t kDecodeMaxWs = 2u << 20;     // partials: at most 2 MiB
constexpr int kDecodeMaxSplit = 256;

struct DecodeArgs {
    int64_t M;
    int num_kb;  // K / 64
    int kbps;    // k-blocks per CTA
    float* ws;   // [nsplit][M][256] partial logits
};

template <bool B_MN>
__global__ void __launch_bounds__(kDThreads, 1)
    fused_decode_proj_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             DecodeArgs da) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = ptx::smem_align<1024>(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kDStages * kDStageBytes);
    uint64_t* empty = full + kDStages;
    uint64_t* accum = empty + kDStages;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accum + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x / kDSlices;
    const int n0 = (blockIdx.x % kDSlices) * kDBN;  // first expert of this CTA's slice
    const int kb0 = split * da.kbps;
    int nkb = da.num_kb - kb0;
    if (nkb > da.kbps) nkb = da.kbps;
    if (nkb < 0) nkb = 0;

    ptx::griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kDStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(accum, 1);
        *s_abort = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, kDBN);
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
                const int s = kb % kDStages;
                if (!ptx::mbar_wait(&empty[s], ((kb / kDStages) & 1) ^ 1, kDWaitNs)) {
                    *s_abort = 1;
                    atomicAdd(&g_watchdog_trips_decode, 1u);
                    break;
                }
                uint8_t* a_s = smem + (size_t)s * kDStageBytes;
                uint8_t* b_s = a_s + kDABytes;
                const int kc = (kb0 + kb) * kDBK;
                ptx::mbar_arrive_expect_tx(&full[s], kDStageBytes);
                ptx::tma_load_2d(a_s, &tmA, kc, 0, &full[s], pol_a);
                if constexpr (B_MN)
                    ptx::tma_load_2d(b_s, &tmB, n0, kc, &full[s], pol_b);  // 64 experts x 64 k, MN-major
                else
                    ptx::tma_load_2d(b_s, &tmB, kc, n0, &full[s], pol_b);  // 64 experts x 64 k, K-major
            }
            // leave only once the copies issued have landed (bounded)
            for (int k = 0; k < kDStages && k < kb; ++k) {
                const int j = kb - 1 - k;
                ptx::mbar_wait(&full[j % kDStages], (j / kDStages) & 1, kDWaitNs);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && nkb > 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kDBM, kDBN, B_MN);
            for (int kb = 0; kb < nkb && !*s_abort; ++kb) {
                const int s = kb % kDStages;
                if (!ptx::mbar_wait(&full[s], (kb / kDStages) & 1, kDWaitNs)) {
                    *s_abort = 1;
                    atomicAdd(&g_watchdog_trips_decode, 1u);
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t a_addr = ptx::smem_u32(smem + (size_t)s * kDStageBytes);
                const uint32_t b_addr = a_addr + kDABytes;
#pragma unroll
                for (int kk = 0; kk < kDBK / 16; ++kk) {
                    const uint64_t adesc = ptx::sdesc_sw128(a_addr + kk * 32, 16, 1024);
                    const uint64_t bdesc = B_MN ? ptx::sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                                : ptx::sdesc_sw128(b_addr + kk * 32, 16, 1024);
                    ptx::umma_bf16(tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                }
                ptx::umma_commit(&empty[s]);
            }
            ptx::umma_commit(accum);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        if (nkb > 0 && !ptx::mbar_wait(accum, 0, kDWaitNs)) {
            if (lane == 0) atomicAdd(&g_watchdog_trips_decode, 1u);
            *s_abort = 1;
        }
        ptx::tc_fence_after();
        const int q = warp & 3;  // TMEM lane quarter of this warp
        const int r = q * 32 + lane;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
        // A timed-out wait leaves NaN partials: the routing kernel then has
        // no valid logits for the batch, and the watchdog counts the event.
        const bool bad = *s_abort != 0;
        if (__any_sync(kFullMask, r < da.M)) {
            float* dst = da.ws + ((size_t)split * da.M + r) * kDE + n0;
#pragma unroll 1
            for (int c0 = 0; c0 < kDBN; c0 += 64) {
                float v[64];
                __syncwarp();
                if (nkb > 0) {
                    ptx::tmem_ld64(t_row + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i) v[i] = 0.0f;
                }
                if (r < da.M) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        reinterpret_cast<float4*>(dst + c0)[i] =
                            bad ? make_float4(NAN, NAN, NAN, NAN)
                                : make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kDBN);
    }
}

// Shape of the split: about kDecodeKbPerCta k-blocks per CTA, the partials
// within kDecodeMaxWs, and no CTA without k-blocks.
void decode_split(int64_t M, int num_kb, int* nsplit, int* kbps) {
    int target = (num_kb + kDecodeKbPerCta - 1) / kDecodeKbPerCta;
    const int64_t cap = (int64_t)(kDecodeMaxWs / ((size_t)M * kDE * sizeof(float)));
    if (target > cap) target = (int)cap;
    if (target > kDecodeMaxSplit) target = kDecodeMaxSplit;
    if (target < 1) target = 1;
    const int per = (num_kb + target - 1) / target;
    *kbps = per;
    *nsplit = (num_kb + per - 1) / per;
}

int set_kernel_smem(const void* fn, size_t bytes, const char* what) {
    static std::mutex mu;
    static std::unordered_map<const void*, std::unordered_map<int, bool>> done;  // kernel -> device -> set
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return set_cuda_error(err, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(mu);
    if (!done[fn][dev]) {
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (err != cudaSuccess) return set_cuda_error(err, what);
        done[fn][dev] = true;
    }
    return MOE_OK;
}

template <bool BIAS, bool GROUPED>
int launch_decode_route(const RouteArgs& ra, cudaStream_t st) {
    auto kern = route_warp_kernel<float, 256, kSigmoid, BIAS, GROUPED, true>;
    const int64_t blocks = ra.M;  // one row per block (M <= 128)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3((unsigned)kWarpRowThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, ra);
    if (err != cudaSuccess) return set_cuda_error(err, "fused router (decode) routing launch");
    return MOE_OK;
}

}  // namespace

size_t fused_decode_workspace_bytes(int64_t M, int num_kb) {
    int nsplit = 1, kbps = 1;
    decode_split(M, num_kb, &nsplit, &kbps);
    return (size_t)nsplit * (size_t)M * kDE * sizeof(float);
}

int launch_fused_decode(const CUtensorMap& tmA, const void* router_weight, bool b_mn, const RouteArgs& route,
                        float* logits_out, int num_kb, void* workspace, cudaStream_t st) {
    int nsplit = 1, kbps = 1;
    decode_split(route.M, num_kb, &nsplit, &kbps);
    // the weight in 64 x 64 boxes: (K, E) rows of 64 experts, or (E, K) rows of 64 k
    const uint64_t K = (uint64_t)num_kb * kDBK;
    CUtensorMap tmB;
    cudaError_t terr = b_mn ? encode_tmap_2d(&tmB, router_weight, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, kDE,
                                             (uint64_t)kDE * 2, 64, kDBK, true)
                            : encode_tmap_2d(&tmB, router_weight, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kDE, K, K * 2,
                                             kDBK, kDBN, true);
    if (terr != cudaSuccess) return set_cuda_error(terr, "cuTensorMapEncodeTiled(router_weight, decode)");
    DecodeArgs da;
    da.M = route.M;
    da.num_kb = num_kb;
    da.kbps = kbps;
    da.ws = static_cast<float*>(workspace);
    {
        const void* fn = b_mn ? reinterpret_cast<const void*>(fused_decode_proj_kernel<true>)
                              : reinterpret_cast<const void*>(fused_decode_proj_kernel<false>);
        int rc = set_kernel_smem(fn, kDSmem, "cudaFuncSetAttribute(fused router decode smem)");
        if (rc != MOE_OK) return rc;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(nsplit * kDSlices), 1, 1);
        cfg.blockDim = dim3(kDThreads, 1, 1);
        cfg.dynamicSmemBytes = kDSmem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t err = b_mn ? cudaLaunchKernelEx(&cfg, fused_decode_proj_kernel<true>, tmA, tmB, da)
                               : cudaLaunchKernelEx(&cfg, fused_decode_proj_kernel<false>, tmA, tmB, da);
        if (err != cudaSuccess) return set_cuda_error(err, "fused router (decode) projection launch");
    }
    RouteArgs ra = route;
    ra.logits = workspace;
    ra.nparts = nsplit;
    ra.part_stride = route.M * kDE;
    ra.logits_out = logits_out;
    const bool grouped = ra.G > 1 && ra.TG < ra.G;
    if (ra.bias)
        return grouped ? launch_decode_route<true, true>(ra, st) : launch_decode_route<true, false>(ra, st);
    return grouped ? launch_decode_route<false, true>(ra, st) : launch_decode_route<false, false>(ra, st);
}

int read_decode_watchdog(unsigned int* count) {
    unsigned int v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_watchdog_trips_decode, sizeof(v));
    if (err != cudaSuccess) return set_cuda_error(err, "cudaMemcpyFromSymbol(decode watchdog)");
    *count = v;
    return MOE_OK;
}

}  // namespace moe
