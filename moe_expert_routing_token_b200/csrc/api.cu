// C ABI of libmoe_routing: argument validation, kernel choice and launch.
//
// Calls follow the signatures of the SGLang routing pages: fused_topk /
// topk_softmax (softmax top-k), grouped_topk_gpu (grouped top-k),
// biased_grouped_topk_impl and aiter_biased_grouped_topk (sigmoid +
// correction_bias), FusedMoeRouter (router projection + routing).  Nothing
// here allocates, synchronises or prints, so every call can be captured in a
// CUDA graph.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "fused_router.cuh"
#include "moe_routing.h"
#include "routing_direct.cuh"
#include "routing_kernels.cuh"
#include "routing_staged.cuh"
#include "routing_stream.cuh"
#include "routing_warp.cuh"
#include "tma_host.cuh"

namespace moe {

namespace {

thread_local char g_last_error[512] = "no error";

int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return status;
}

int cuda_fail(cudaError_t err, const char* what) {
    return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(err), cudaGetErrorString(err));
}

// Per-device SM count and per-kernel residency, looked up once.
struct LaunchCache {
    std::mutex mu;
    std::unordered_map<int, int> sms;
    std::unordered_map<int, std::unordered_map<const void*, int>> per_sm;  // device -> kernel -> blocks
};
LaunchCache& cache() {
    static LaunchCache c;
    return c;
}

int device_and_sms(int* dev, int* sms) {
    cudaError_t err = cudaGetDevice(dev);
    if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
    LaunchCache& c = cache();
    std::lock_guard<std::mutex> lk(c.mu);
    auto it = c.sms.find(*dev);
    if (it != c.sms.end()) {
        *sms = it->second;
        return MOE_OK;
    }
    int n = 0;
    err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, *dev);
    if (err != cudaSuccess) return cuda_fail(err, "cudaDeviceGetAttribute");
    c.sms[*dev] = n;
    *sms = n;
    return MOE_OK;
}

template <typename Kernel>
int resident_blocks(int dev, Kernel k, int threads, size_t smem, int* out) {
    LaunchCache& c = cache();
    const void* key = reinterpret_cast<const void*>(k);
    std::lock_guard<std::mutex> lk(c.mu);
    auto& m = c.per_sm[dev];
    auto it = m.find(key);
    if (it != m.end()) {
        *out = it->second;
        return MOE_OK;
    }
    int n = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem);
    if (err != cudaSuccess) return cuda_fail(err, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (n < 1) n = 1;
    m[key] = n;
    *out = n;
    return MOE_OK;
}

// Persistent-style grid: enough blocks for the work, capped at one full wave
// of resident blocks over all SMs.
template <typename Kernel>
int launch_rows(Kernel k, int threads, size_t smem, int64_t rows_per_block, const RouteArgs& a,
                cudaStream_t stream) {
    int dev = 0, sms = 0, per_sm = 1;
    int rc = device_and_sms(&dev, &sms);
    if (rc != MOE_OK) return rc;
    rc = resident_blocks(dev, k, threads, smem, &per_sm);
    if (rc != MOE_OK) return rc;
    const int64_t need = (a.M + rows_per_block - 1) / rows_per_block;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    k<<<grid, threads, smem, stream>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "routing kernel launch");
    return MOE_OK;
}

bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

// Experts per lane for E = 256 (32: 8 lanes per row; 16: 16 lanes per row).
#ifndef MOE_SEG_C256
#define MOE_SEG_C256 32
#endif
constexpr int kC256 = MOE_SEG_C256;

template <typename TIn, int SCORE, bool BIAS>
int launch_segment(int E, const RouteArgs& a, cudaStream_t st) {
    if (E == 256) {
        constexpr int L = 256 / kC256, R = 32 / L;
        return launch_rows(route_segment_kernel<TIn, 256, kC256, SCORE, BIAS>, kSegThreads, 0,
                           (kSegThreads / 32) * R, a, st);
    }
    constexpr int L = 160 / 20, R = 32 / L;
    return launch_rows(route_segment_kernel<TIn, 160, 20, SCORE, BIAS>, kSegThreads, 0,
                       (kSegThreads / 32) * R, a, st);
}

// Batches at least this large take the TMA-staged streaming kernel.
constexpr int64_t kStagedMinRows = 1024;

// Launch a persistent TMA-ring routing kernel: raise its dynamic shared
// memory limit once per (kernel, device), encode the logits tensor map
// (boxes of box_e x rb elements, 128-byte swizzle) and size the grid to the
// resident blocks.
using RingKernel = void (*)(const CUtensorMap, RouteArgs, int64_t);

template <typename TIn>
int launch_ring(RingKernel kern, size_t smem, int threads, int box_e, int rb, const RouteArgs& a,
                cudaStream_t st, const char* what) {
    int dev = 0, sms = 0, per_sm = 1;
    int rc = device_and_sms(&dev, &sms);
    if (rc != MOE_OK) return rc;
    {
        static std::mutex mu;
        static std::unordered_map<int, std::unordered_map<const void*, bool>> done;  // device -> kernel -> set
        std::lock_guard<std::mutex> lk(mu);
        bool& set = done[dev][reinterpret_cast<const void*>(kern)];
        if (!set) {
            cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (err != cudaSuccess) return cuda_fail(err, what);
            set = true;
        }
    }
    rc = resident_blocks(dev, kern, threads, smem, &per_sm);
    if (rc != MOE_OK) return rc;
    CUtensorMap tmap;
    cudaError_t err = encode_tmap_2d(&tmap, a.logits,
                                     sizeof(TIn) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                                     (uint64_t)a.M, (uint64_t)a.E, (uint64_t)a.E * sizeof(TIn), box_e, rb, true);
    if (err != cudaSuccess) return cuda_fail(err, "cuTensorMapEncodeTiled(logits)");
    const int64_t nblocks = (a.M + rb - 1) / rb;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(nblocks < cap ? nblocks : cap);
    // Programmatic dependent launch: the block's prologue (barrier set-up,
    // descriptor prefetch) overlaps the previous kernel in the stream; the
    // kernel waits for that kernel (griddepcontrol.wait) before it touches any
    // input or output.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, tmap, a, nblocks);
    if (err != cudaSuccess) return cuda_fail(err, what);
    return MOE_OK;
}

template <typename TIn, int E, int C, int SCORE, bool BIAS>
int launch_staged_ec(const RouteArgs& a, cudaStream_t st) {
    using Cfg = StagedCfg<TIn, E, C, SCORE, BIAS>;
    return launch_ring<TIn>(route_staged_kernel<TIn, E, C, SCORE, BIAS>, Cfg::SMEM, (Cfg::W + 1) * 32,
                            Cfg::BOX_E, Cfg::RB, a, st, "staged routing kernel");
}

template <typename TIn, int E, int C, int SCORE, bool BIAS, bool APPROX>
int launch_stream_ec(const RouteArgs& a, cudaStream_t st) {
    using Cfg = StreamCfg<TIn, E, C, SCORE, BIAS, APPROX>;
    return launch_ring<TIn>(route_stream_kernel<TIn, E, C, SCORE, BIAS, APPROX>, Cfg::SMEM,
                            kStreamThreads, Cfg::BOX_E, Cfg::RB, a, st, "streaming routing kernel");
}

// Two-phase streaming kernel (topk <= 8).  The approximate phase-1 key is
// used for sigmoid scoring when every group is kept.
template <typename TIn, int SCORE, bool BIAS>
int launch_stream(int E, const RouteArgs& a, cudaStream_t st) {
    const bool approx = (SCORE == kSigmoid) && a.TG == a.G;
    if (E == 256)
        return approx ? launch_stream_ec<TIn, 256, 32, SCORE, BIAS, SCORE == kSigmoid>(a, st)
                      : launch_stream_ec<TIn, 256, 32, SCORE, BIAS, false>(a, st);
    return approx ? launch_stream_ec<TIn, 160, 20, SCORE, BIAS, SCORE == kSigmoid>(a, st)
                  : launch_stream_ec<TIn, 160, 20, SCORE, BIAS, false>(a, st);
}

template <typename TIn, int SCORE, bool BIAS>
int launch_staged(int E, const RouteArgs& a, cudaStream_t st) {
    if (E == 256) return launch_staged_ec<TIn, 256, kC256, SCORE, BIAS>(a, st);
    return launch_staged_ec<TIn, 160, 20, SCORE, BIAS>(a, st);
}

template <typename TIn, int SCORE, bool BIAS>
int launch_small(int E, const RouteArgs& a, cudaStream_t st) {
    switch (E) {
        case 8: return launch_rows(route_small_kernel<TIn, 8, SCORE, BIAS>, 256, 0, 256, a, st);
        case 16: return launch_rows(route_small_kernel<TIn, 16, SCORE, BIAS>, 256, 0, 256, a, st);
        default: return launch_rows(route_small_kernel<TIn, 32, SCORE, BIAS>, 256, 0, 256, a, st);
    }
}

template <typename TIn, int SCORE>
int launch_generic(const RouteArgs& a, cudaStream_t st) {
    const int per_warp = generic_smem_per_warp(a.E, a.G);
    int warps = (48 * 1024) / per_warp;
    if (warps > 4) warps = 4;
    if (warps < 1) return fail(MOE_ERR_UNSUPPORTED, "E=%d, G=%d need too much shared memory", a.E, a.G);
    return launch_rows(route_generic_kernel<TIn, SCORE>, warps * 32, (size_t)warps * per_warp,
                       warps, a, st);
}

// Direct kernel: raise its dynamic shared memory limit once per device, size
// the grid to the octets (R rows per warp) capped at one wave of resident
// blocks, and launch with programmatic dependent launch (the kernel waits for
// the previous kernel before it reads any input).
template <typename TIn, int E, int L, int SCORE, bool BIAS, int MODE, int GS>
int launch_direct(const RouteArgs& a, cudaStream_t st) {
    auto kern = route_direct_kernel<TIn, E, L, SCORE, BIAS, MODE, GS>;
    constexpr size_t smem = direct_smem_bytes<TIn, E, L>();
    int dev = 0, sms = 0, per_sm = 1;
    int rc = device_and_sms(&dev, &sms);
    if (rc != MOE_OK) return rc;
    {
        static std::mutex mu;
        static std::unordered_map<int, bool> done;  // device ordinal -> attribute set
        std::lock_guard<std::mutex> lk(mu);
        if (!done[dev]) {
            cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (err != cudaSuccess) return cuda_fail(err, "direct routing kernel attribute");
            done[dev] = true;
        }
    }
    rc = resident_blocks(dev, kern, kDirectThreads, smem, &per_sm);
    if (rc != MOE_OK) return rc;
    using Shape = DirectShape<TIn, E, L>;
    constexpr int R = Shape::R;
    const int64_t n_oct = (a.M + R - 1) / R;
    // E = 256: the logits seen as rows of 128 bytes, one box of R token rows
    // per copy, 128-byte swizzle
    CUtensorMap tmap;
    memset(&tmap, 0, sizeof(tmap));
    if constexpr (Shape::TMA) {
        cudaError_t err = encode_tmap_2d(&tmap, a.logits,
                                         sizeof(TIn) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                                         (uint64_t)a.M * Shape::TROWS, 128 / sizeof(TIn), 128, 128 / sizeof(TIn),
                                         R * Shape::TROWS, true);
        if (err != cudaSuccess) return cuda_fail(err, "cuTensorMapEncodeTiled(logits)");
    }
    const int64_t need = (n_oct + kDirectWarps - 1) / kDirectWarps;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3((unsigned)kDirectThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, tmap, a, n_oct);
    if (err != cudaSuccess) return cuda_fail(err, "direct routing kernel launch");
    return MOE_OK;
}

// Batches up to this size route one row per warp (route_warp_kernel): the
// shortest chain per row.  Where the direct kernel takes the shape (E = 256,
// k <= 8, every group kept or 8 groups) it takes over above 3072 rows:
// measured on B200 (bf16 E = 256, k = 8, sigmoid with bias), the warp-per-row
// kernel takes 2.1 / 2.5 / 3.1 us at M = 256 / 1024 / 2048 against 2.8 / 3.4
// / 3.5 for the direct kernel, and 4.7 against 4.4 us at M = 4096 (grouped,
// G = 8: 5.3 against 4.8).
constexpr int64_t kWarpRowMaxRows = 4096;
constexpr int64_t kWarpRowMaxRowsBeforeDirect = 3072;

template <typename TIn, int E, int SCORE, bool BIAS, bool GROUPED>
int launch_warp_rows(const RouteArgs& a, cudaStream_t st) {
    auto kern = route_warp_kernel<TIn, E, SCORE, BIAS, GROUPED>;
    int dev = 0, sms = 0;
    int rc = device_and_sms(&dev, &sms);
    if (rc != MOE_OK) return rc;
    const int64_t need = (a.M + kWarpRowWarps - 1) / kWarpRowWarps;
    const int64_t cap = (int64_t)sms * 16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(need < cap ? need : cap), 1, 1);
    cfg.blockDim = dim3((unsigned)kWarpRowThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, a);
    if (err != cudaSuccess) return cuda_fail(err, "warp-per-row routing kernel launch");
    return MOE_OK;
}

// The warp-per-row kernel's shapes: E = 256 or 160 (C = E / 32 experts per
// lane), groups of whole lanes (G divides 32), decode-sized batches; 16-byte
// aligned rows where a lane's segment is read with 16-byte loads.  Returns -1
// otherwise.
template <typename TIn, int E, int SCORE, bool BIAS>
int try_warp_rows_e(const RouteArgs& a, cudaStream_t st) {
    constexpr int SEGB = (E / 32) * (int)sizeof(TIn);
    if (SEGB % 16 == 0 && !aligned(a.logits, 16)) return -1;
    if (a.G > 1 && a.TG < a.G) return launch_warp_rows<TIn, E, SCORE, BIAS, true>(a, st);
    return launch_warp_rows<TIn, E, SCORE, BIAS, false>(a, st);
}

template <typename TIn, int SCORE, bool BIAS>
int try_warp_rows(const RouteArgs& a, cudaStream_t st) {
    // the shapes try_direct takes (below its row limit)
    const bool direct_shape = a.E == 256 && a.K <= 8 && (a.TG == a.G || a.G == 8) && aligned(a.logits, 16);
    if (a.M > (direct_shape ? kWarpRowMaxRowsBeforeDirect : kWarpRowMaxRows) || 32 % a.G != 0) return -1;
    if (a.E == 256) return try_warp_rows_e<TIn, 256, SCORE, BIAS>(a, st);
    if (a.E == 160) return try_warp_rows_e<TIn, 160, SCORE, BIAS>(a, st);
    return -1;
}

// The direct kernel's shapes (instantiated for E = 256; try_direct keeps
// E = 160 off it): topk <= 8, every group kept or 8 groups.  Returns -1 for
// other shapes.
template <typename TIn, int E, int L, int SCORE, bool BIAS>
int try_direct_el(const RouteArgs& a, cudaStream_t st) {
    constexpr int GS8 = E / 8;  // experts per group with 8 groups
    if (a.TG == a.G) {
        if constexpr (SCORE == kSigmoid && BIAS) return launch_direct<TIn, E, L, SCORE, BIAS, kKeyApprox, 0>(a, st);
        else return launch_direct<TIn, E, L, SCORE, BIAS, kKeyRaw, 0>(a, st);
    }
    if (a.G == 8) {
        constexpr int MODE = SCORE == kSigmoid ? kKeyExact : kKeyRaw;
        return launch_direct<TIn, E, L, SCORE, BIAS, MODE, GS8>(a, st);
    }
    return -1;
}

// Eight lanes per row at every batch size.  Measured on B200 (bf16 E = 256,
// k = 8, sigmoid with bias): 10.7 / 18.7 us at M = 32768 / 65536 against
// 11.7 / 19.5 with 4 lanes per row (grouped, G = 8: 13.9 / 25.1 against
// 15.8 / 27.4).  The four-lane form issues fewer instructions per row but
// runs half the warps with twice the serial work each.
template <typename TIn, int E, int SCORE, bool BIAS>
int try_direct_e(const RouteArgs& a, cudaStream_t st) {
    return try_direct_el<TIn, E, 8, SCORE, BIAS>(a, st);
}

// Above this many rows the two-phase streaming kernel, whose ring keeps every
// SM busy for the whole call, issues fewer instructions per row and wins.
// Measured on B200 (bf16 E = 256, k = 8): 33.9 against 36.9 us at M = 131072
// and 58.8 against 69.2 at 262144 (sigmoid with bias); grouped (G = 8,
// TG = 4) 40.0 against 50.3 and 70.2 against 96.8.
constexpr int64_t kDirectMaxRows = 65536;
constexpr int64_t kDirectMaxRows160 = 16384;

template <typename TIn, int SCORE, bool BIAS>
int try_direct(const RouteArgs& a, cudaStream_t st) {
    if (a.K > 8 || !aligned(a.logits, 16) || a.M > kDirectMaxRows) return -1;
    if (a.E == 256) return try_direct_e<TIn, 256, SCORE, BIAS>(a, st);
    // fp32 E = 160 (rows staged by per-row copies, 20 experts per lane) up to
    // 16384 rows; above, the two-phase streaming kernel.  Measured on B200
    // (softmax, G = 8, TG = 3, k = 6): 5.7 / 9.3 / 15.0 us at M = 8192 /
    // 16384 / 32768 against 7.7 / 9.6 / 13.8 for the streaming kernel.
    if constexpr (sizeof(TIn) == 4)
        if (a.E == 160 && a.M <= kDirectMaxRows160) return try_direct_e<TIn, 160, SCORE, BIAS>(a, st);
    return -1;
}

template <typename TIn, int SCORE, bool BIAS>
int dispatch_typed(const RouteArgs& a, cudaStream_t st) {
    const int E = a.E;
    {
        const int rc = try_warp_rows<TIn, SCORE, BIAS>(a, st);
        if (rc >= 0) return rc;
    }
    {
        const int rc = try_direct<TIn, SCORE, BIAS>(a, st);
        if (rc >= 0) return rc;
    }
    const size_t esz = sizeof(TIn);
    if ((E == 256 || E == 160) && (E == 256 ? 256 / kC256 : 8) % a.G == 0) {
        const int C = (E == 256) ? kC256 : 20;
        const size_t chunk = C * esz;
        const size_t vec = (chunk % 16 == 0) ? 16 : 8;
        if (a.M >= kStagedMinRows && aligned(a.logits, 16) && (E * esz) % 16 == 0)
            return (a.K <= 8 && (E == 160 || kC256 == 32)) ? launch_stream<TIn, SCORE, BIAS>(E, a, st)
                                                          : launch_staged<TIn, SCORE, BIAS>(E, a, st);
        if (aligned(a.logits, vec)) return launch_segment<TIn, SCORE, BIAS>(E, a, st);
    }
    if ((E == 8 || E == 16 || E == 32) && aligned(a.logits, 16))
        return launch_small<TIn, SCORE, BIAS>(E, a, st);
    return launch_generic<TIn, SCORE>(a, st);
}

int route(const void* logits, int dtype, const float* bias, int64_t M, int E, int K, int renorm,
          int G, int TG, int group_kind, int scoring, float rsf, float* weights, int32_t* ids,
          void* stream, const char* who, int bias_bf16 = 0, float softcap = 0.0f) {
    if (dtype != MOE_DTYPE_F32 && dtype != MOE_DTYPE_BF16)
        return fail(MOE_ERR_INVALID_ARG, "%s: dtype %d is neither MOE_DTYPE_F32 nor MOE_DTYPE_BF16", who, dtype);
    if (M < 0) return fail(MOE_ERR_INVALID_ARG, "%s: M=%lld < 0", who, (long long)M);
    if (E < 1) return fail(MOE_ERR_INVALID_ARG, "%s: E=%d < 1", who, E);
    if (G < 1 || E % G != 0)
        return fail(MOE_ERR_INVALID_ARG, "%s: num_expert_group=%d does not divide E=%d", who, G, E);
    if (TG < 1 || TG > G)
        return fail(MOE_ERR_INVALID_ARG, "%s: topk_group=%d outside [1, %d]", who, TG, G);
    if (K < 1 || K > TG * (E / G))
        return fail(MOE_ERR_INVALID_ARG, "%s: topk=%d outside [1, topk_group*E/G=%d]", who, K, TG * (E / G));
    if (!std::isfinite(rsf)) return fail(MOE_ERR_INVALID_ARG, "%s: routed_scaling_factor is not finite", who);
    if (!std::isfinite(softcap)) return fail(MOE_ERR_INVALID_ARG, "%s: softcap is not finite", who);
    if (E > 1024) return fail(MOE_ERR_UNSUPPORTED, "%s: E=%d > 1024", who, E);
    if (K > 32) return fail(MOE_ERR_UNSUPPORTED, "%s: topk=%d > 32", who, K);
    if (M == 0) return MOE_OK;
    if (!logits || !weights || !ids) return fail(MOE_ERR_INVALID_ARG, "%s: null pointer argument", who);
    const size_t esz = dtype == MOE_DTYPE_F32 ? 4 : 2;
    if (!aligned(logits, esz) || !aligned(weights, 4) || !aligned(ids, 4) || (bias && !aligned(bias, 4)))
        return fail(MOE_ERR_INVALID_ARG, "%s: pointer not aligned to its element size", who);

    RouteArgs a;
    a.logits = logits;
    a.bias = bias;
    a.M = M;
    a.E = E;
    a.G = G;
    a.TG = TG;
    a.K = K;
    a.group_kind = group_kind;
    a.renorm = renorm ? 1 : 0;
    a.rsf = rsf;
    a.weights = weights;
    a.ids = ids;
    a.bias_bf16 = (bias_bf16 && dtype == MOE_DTYPE_BF16) ? 1 : 0;  // an fp32 cast of fp32 logits changes nothing
    a.softcap = (scoring == kSoftmax) ? softcap : 0.0f;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (scoring == kSoftmax) {
        a.bias = nullptr;
        return dtype == MOE_DTYPE_F32 ? dispatch_typed<float, kSoftmax, false>(a, st)
                                      : dispatch_typed<__nv_bfloat16, kSoftmax, false>(a, st);
    }
    if (bias)
        return dtype == MOE_DTYPE_F32 ? dispatch_typed<float, kSigmoid, true>(a, st)
                                      : dispatch_typed<__nv_bfloat16, kSigmoid, true>(a, st);
    return dtype == MOE_DTYPE_F32 ? dispatch_typed<float, kSigmoid, false>(a, st)
                                  : dispatch_typed<__nv_bfloat16, kSigmoid, false>(a, st);
}

}  // namespace

int read_routing_watchdog(unsigned int* count) {
    unsigned int v = 0, w = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_watchdog_trips_routing, sizeof(v));
    if (err != cudaSuccess) return cuda_fail(err, "cudaMemcpyFromSymbol(watchdog)");
    err = cudaMemcpyFromSymbol(&w, g_watchdog_trips_direct, sizeof(w));
    if (err != cudaSuccess) return cuda_fail(err, "cudaMemcpyFromSymbol(direct watchdog)");
    *count = v + w;
    return MOE_OK;
}

int set_error(int status, const char* msg) { return fail(status, "%s", msg); }
int set_cuda_error(cudaError_t err, const char* what) { return cuda_fail(err, what); }
int sm_count(int* dev, int* sms) { return device_and_sms(dev, sms); }
int route_logits(const void* logits, int dtype, const float* bias, int64_t M, int E, int K,
                 int renorm, int G, int TG, float rsf, float* weights, int32_t* ids, void* stream) {
    return route(logits, dtype, bias, M, E, K, renorm, G, TG, kGroupTop2Sum, kSigmoid, rsf, weights,
                 ids, stream, "moe_fused_router_topk");
}

}  // namespace moe

extern "C" {

int moe_abi_version(void) { return MOE_ROUTING_ABI_VERSION; }

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        default: return "MOE_ERR_UNKNOWN";
    }
}

const char* moe_last_error(void) { return moe::g_last_error; }

int moe_watchdog_trips(unsigned int* count) {
    if (!count) return moe::fail(MOE_ERR_INVALID_ARG, "moe_watchdog_trips: null pointer");
    unsigned int a = 0, b = 0;
    int rc = moe::read_routing_watchdog(&a);
    if (rc != MOE_OK) return rc;
    rc = moe::read_fused_watchdog(&b);
    if (rc != MOE_OK) return rc;
    unsigned int c = 0, d = 0;
    rc = moe::read_top1_watchdog(&c);
    if (rc != MOE_OK) return rc;
    rc = moe::read_decode_watchdog(&d);
    if (rc != MOE_OK) return rc;
    *count = a + b + c + d;
    return MOE_OK;
}

int moe_topk_softmax(const void* gating_output, int dtype, int64_t M, int32_t E, int32_t topk,
                     int32_t renormalize, float* topk_weights, int32_t* topk_ids, void* stream) {
    return moe::route(gating_output, dtype, nullptr, M, E, topk, renormalize, 1, 1, moe::kGroupMax,
                      moe::kSoftmax, 1.0f, topk_weights, topk_ids, stream, "moe_topk_softmax");
}

int moe_grouped_topk(const void* gating_output, int dtype, int64_t M, int32_t E, int32_t topk,
                     int32_t renormalize, int32_t num_expert_group, int32_t topk_group,
                     float routed_scaling_factor, float* topk_weights, int32_t* topk_ids,
                     void* stream) {
    return moe::route(gating_output, dtype, nullptr, M, E, topk, renormalize, num_expert_group,
                      topk_group, moe::kGroupMax, moe::kSoftmax, routed_scaling_factor, topk_weights,
                      topk_ids, stream, "moe_grouped_topk");
}

int moe_biased_grouped_topk(const void* gating_output, int dtype, const float* correction_bias,
                            int64_t M, int32_t E, int32_t topk, int32_t renormalize,
                            int32_t num_expert_group, int32_t topk_group,
                            float routed_scaling_factor, float* topk_weights, int32_t* topk_ids,
                            void* stream) {
    return moe::route(gating_output, dtype, correction_bias, M, E, topk, renormalize,
                      num_expert_group, topk_group, moe::kGroupTop2Sum, moe::kSigmoid,
                      routed_scaling_factor, topk_weights, topk_ids, stream,
                      "moe_biased_grouped_topk");
}

int moe_grouped_topk_softcap(const void* gating_output, int dtype, int64_t M, int32_t E, int32_t topk,
                             int32_t renormalize, int32_t num_expert_group, int32_t topk_group,
                             float routed_scaling_factor, float softcap, float* topk_weights, int32_t* topk_ids,
                             void* stream) {
    return moe::route(gating_output, dtype, nullptr, M, E, topk, renormalize, num_expert_group, topk_group,
                      moe::kGroupMax, moe::kSoftmax, routed_scaling_factor, topk_weights, topk_ids, stream,
                      "moe_grouped_topk_softcap", 0, softcap);
}

int moe_biased_grouped_topk_aiter(const void* gating_output, int dtype, const float* correction_bias,
                                  int64_t M, int32_t E, int32_t topk, int32_t renormalize,
                                  int32_t num_expert_group, int32_t topk_group,
                                  float routed_scaling_factor, float* topk_weights, int32_t* topk_ids,
                                  void* stream) {
    return moe::route(gating_output, dtype, correction_bias, M, E, topk, renormalize,
                      num_expert_group, topk_group, moe::kGroupTop2Sum, moe::kSigmoid,
                      routed_scaling_factor, topk_weights, topk_ids, stream,
                      "moe_biased_grouped_topk_aiter", 1);
}

}  // extern "C"
