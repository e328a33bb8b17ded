// Expert-sorted token permutation of a routing result: the step after top-k
// in the SGLang MoE routing page's structure diagram (구조도), whose "Triton
// Kernels routing" branch hands the expert runner RoutingData, GatherIndx and
// ScatterIndx (출력 포맷: TRITON_KERNEL).  The page shows no body; what is
// computed is a stable counting sort of the M*k (token, slot) pairs of
// topk_ids by expert id, pair index i = token*k + slot:
//   expert_counts[e], expert_offsets[e] (exclusive prefix, [E] = valid pairs),
//   gather_indx[p] = the pair at sorted position p (experts ascending, pairs
//   ascending within an expert), scatter_indx[i] = the position of pair i,
//   gate_scal[p] = topk_weights of gather_indx[p].
//
// Three passes, deterministic (no atomics decide an order):
//   1. perm_hist_kernel: one block per tile of kPermTile pairs counts its
//      experts in shared memory and writes the tile's counts to the workspace.
//   2. perm_scan_kernel: one block of up to 1024 threads (expert x chunk of
//      tiles) turns the [tiles][E] counts into expert totals, offsets, and
//      each tile's first position per expert.
//   3. perm_scatter_kernel: each warp of a tile takes a contiguous run of the
//      tile's pairs in order; within a 32-pair piece, lanes holding the same
//      expert are ranked by __match_any_sync, so pairs keep their index order.
// Ids outside [0, E) are skipped: not counted, scatter_indx = -1.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>

#include "moe_routing.h"

namespace moe {

int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);

namespace {

constexpr int kPermTile = 1024;    // pairs per block
constexpr int kPermThreads = 256;  // 8 warps; each warp owns 128 consecutive pairs of the tile
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermMaxE = 1024;

__global__ void __launch_bounds__(kPermThreads) perm_hist_kernel(const int32_t* __restrict__ ids, int64_t n, int E,
                                                                 int32_t* __restrict__ tile_counts) {
    __shared__ int32_t h[kPermMaxE];
    for (int e = threadIdx.x; e < E; e += kPermThreads) h[e] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * kPermTile;
    for (int j = threadIdx.x; j < kPermTile; j += kPermThreads) {
        const int64_t i = t0 + j;
        if (i < n) {
            const int id = __ldg(ids + i);
            if (id >= 0 && id < E) atomicAdd(&h[id], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kPermThreads) tile_counts[(int64_t)blockIdx.x * E + e] = h[e];
}

// One block of E32 x Q threads (E32 = E rounded up to a warp, Q = 1024 / E32
// chunks of tiles): thread (q, e) sums expert e over its chunk of tiles; the
// chunk sums are prefixed per expert and the expert totals scanned in shared
// memory; then the thread rewrites its chunk's counts as each tile's first
// position of expert e.
__global__ void __launch_bounds__(kPermMaxE) perm_scan_kernel(int32_t* __restrict__ tile_counts, int ntiles, int E,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ offsets) {
    __shared__ int32_t part[kPermMaxE];  // [Q][E32]: chunk sums, then each chunk's first position
    __shared__ int32_t warp_sum[32];
    __shared__ int32_t total;
    const int E32 = (E + 31) & ~31;
    const int Q = blockDim.x / E32;
    const int e = threadIdx.x % E32, q = threadIdx.x / E32;
    const int per = (ntiles + Q - 1) / Q;
    const int b0 = q * per, b1 = min(ntiles, b0 + per);
    int32_t s = 0;
    if (e < E) {
#pragma unroll 8
        for (int b = b0; b < b1; ++b) s += tile_counts[(int64_t)b * E + e];
    }
    part[q * E32 + e] = s;
    __syncthreads();
    // chunk-0 threads (the first E32 threads, whole warps): prefix over the
    // chunks of their expert, then an exclusive scan of the expert totals
    int32_t excl = 0, cnt = 0;
    if (q == 0) {
        for (int c = 0; c < Q; ++c) {
            const int32_t v = part[c * E32 + e];
            part[c * E32 + e] = cnt;
            cnt += v;
        }
        if (e >= E) cnt = 0;
        const int lane = e & 31;
        int32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) warp_sum[e >> 5] = incl;
        excl = incl - cnt;
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // scan of the warp totals
        const int nw = E32 >> 5;
        const int lane = threadIdx.x;
        const int32_t v = lane < nw ? warp_sum[lane] : 0;
        int32_t vi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, vi, o);
            if (lane >= o) vi += t;
        }
        if (lane < nw) warp_sum[lane] = vi - v;
        if (lane == nw - 1) total = vi;
    }
    __syncthreads();
    if (q == 0 && e < E) {
        const int32_t off = warp_sum[e >> 5] + excl;
        counts[e] = cnt;
        offsets[e] = off;
        for (int c = 0; c < Q; ++c) part[c * E32 + e] += off;
    }
    if (threadIdx.x == 0) offsets[E] = total;
    __syncthreads();
    if (e < E) {
        int32_t run = part[q * E32 + e];
#pragma unroll 8
        for (int b = b0; b < b1; ++b) {
            int32_t* p = tile_counts + (int64_t)b * E + e;
            const int32_t v = *p;
            *p = run;
            run += v;
        }
    }
}

__global__ void __launch_bounds__(kPermThreads)
    perm_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ weights, int64_t n, int E,
                        const int32_t* __restrict__ tile_base, int32_t* __restrict__ gather,
                        int32_t* __restrict__ scatter, float* __restrict__ gate) {
    extern __shared__ int32_t wbase[];  // [kPermWarps][E]: next position per (warp, expert)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kRun = kPermTile / kPermWarps;  // pairs per warp
    const int64_t t0 = (int64_t)blockIdx.x * kPermTile;
    const int64_t w0 = t0 + (int64_t)warp * kRun;
    for (int e = threadIdx.x; e < kPermWarps * E; e += kPermThreads) wbase[e] = 0;
    __syncthreads();
    // per-warp counts
    for (int j = lane; j < kRun; j += 32) {
        const int64_t i = w0 + j;
        if (i < n) {
            const int id = __ldg(ids + i);
            if (id >= 0 && id < E) atomicAdd(&wbase[warp * E + id], 1);
        }
    }
    __syncthreads();
    // exclusive prefix over the warps of the tile, from the tile's base
    for (int e = threadIdx.x; e < E; e += kPermThreads) {
        int32_t run = tile_base[(int64_t)blockIdx.x * E + e];
        for (int w = 0; w < kPermWarps; ++w) {
            const int32_t c = wbase[w * E + e];
            wbase[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    // place the warp's pairs in order, 32 at a time
    const unsigned lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < kRun; j0 += 32) {
        const int64_t i = w0 + j0 + lane;
        int id = -1;
        if (i < n) {
            id = __ldg(ids + i);
            if (id < 0 || id >= E) {
                scatter[i] = -1;
                id = -1;
            }
        }
        const unsigned same = __match_any_sync(0xffffffffu, id);
        int32_t pos = 0;
        if (id >= 0) pos = wbase[warp * E + id] + __popc(same & lt);
        __syncwarp();
        if (id >= 0) {
            gather[pos] = (int32_t)i;
            scatter[i] = pos;
            if (gate) gate[pos] = __ldg(weights + i);
            if ((same >> lane) == 1u) wbase[warp * E + id] = pos + 1;  // the group's last lane
        }
        __syncwarp();
    }
}

int64_t perm_tiles(int64_t n) { return (n + kPermTile - 1) / kPermTile; }

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_expert_permutation_workspace_size(int64_t M, int32_t k, int32_t E) {
    if (M < 0 || k < 1 || E < 1 || E > moe::kPermMaxE) return (size_t)-1;
    if (M >= ((int64_t)1 << 31)) return (size_t)-1;  // M * k below: no overflow
    const int64_t n = M * (int64_t)k;
    if (n >= ((int64_t)1 << 31)) return (size_t)-1;
    return (size_t)(moe::perm_tiles(n) * E * (int64_t)sizeof(int32_t));
}

int moe_expert_permutation(const int32_t* topk_ids, const float* topk_weights, int64_t M, int32_t k, int32_t E,
                           int32_t* expert_counts, int32_t* expert_offsets, int32_t* gather_indx,
                           int32_t* scatter_indx, float* gate_scal, void* workspace, size_t workspace_bytes,
                           void* stream) {
    using namespace moe;
    char msg[256];
    if (M < 0 || k < 1 || E < 1) {
        std::snprintf(msg, sizeof msg, "moe_expert_permutation: bad sizes M=%lld k=%d E=%d", (long long)M, k, E);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (E > kPermMaxE) {
        std::snprintf(msg, sizeof msg, "moe_expert_permutation: E=%d > %d", E, kPermMaxE);
        return set_error(MOE_ERR_UNSUPPORTED, msg);
    }
    if (M >= ((int64_t)1 << 31) || M * (int64_t)k >= ((int64_t)1 << 31))
        return set_error(MOE_ERR_UNSUPPORTED, "moe_expert_permutation: M*k >= 2^31");
    const int64_t n = M * (int64_t)k;
    if (!expert_counts || !expert_offsets)
        return set_error(MOE_ERR_INVALID_ARG, "moe_expert_permutation: null counts or offsets");
    if (n > 0 && (!topk_ids || !gather_indx || !scatter_indx))
        return set_error(MOE_ERR_INVALID_ARG, "moe_expert_permutation: null pointer argument");
    if ((gate_scal != nullptr) != (topk_weights != nullptr))
        return set_error(MOE_ERR_INVALID_ARG,
                         "moe_expert_permutation: topk_weights and gate_scal must both be given or both be null");
    const size_t need = moe_expert_permutation_workspace_size(M, k, E);
    if (n > 0 && (workspace == nullptr || workspace_bytes < need)) {
        std::snprintf(msg, sizeof msg, "moe_expert_permutation: workspace of %zu bytes needed, %zu given", need,
                      workspace_bytes);
        return set_error(MOE_ERR_INVALID_ARG, msg);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n == 0) {
        cudaError_t err = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, st);
        if (err == cudaSuccess) err = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), st);
        return err == cudaSuccess ? MOE_OK : set_cuda_error(err, "moe_expert_permutation: memset");
    }
    int32_t* tiles = static_cast<int32_t*>(workspace);
    const int ntiles = (int)perm_tiles(n);
    perm_hist_kernel<<<ntiles, kPermThreads, 0, st>>>(topk_ids, n, E, tiles);
    const int e32 = ((E + 31) / 32) * 32;
    perm_scan_kernel<<<1, e32 * (kPermMaxE / e32), 0, st>>>(tiles, ntiles, E, expert_counts, expert_offsets);
    perm_scatter_kernel<<<ntiles, kPermThreads, sizeof(int32_t) * kPermWarps * E, st>>>(
        topk_ids, topk_weights, n, E, tiles, gather_indx, scatter_indx, gate_scal);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_cuda_error(err, "moe_expert_permutation: launch");
    return MOE_OK;
}

}  // extern "C"
