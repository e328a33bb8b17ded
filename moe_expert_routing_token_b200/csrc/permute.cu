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
// Two launches, deterministic (no atomic decides an order):
//   1. perm_count_kernel: one block per tile of kPermTile pairs counts its
//      experts in shared memory and writes the tile's counts to the
//      workspace ([tiles][E] int32).
//   2. perm_place_kernel (programmatic dependent launch: its set-up overlaps
//      the first): every block sums, per expert, the counts of the tiles
//      before its own and of all tiles (coalesced reads of the workspace, which
//      sits in L2), scans the totals over the experts for the offsets, adds
//      its warps' counts in warp order, and places its pairs: each warp takes
//      a contiguous run of the tile's pairs in order; within a 32-pair piece,
//      lanes holding the same expert are ranked by __match_any_sync, so pairs
//      keep their index order.  Block 0 writes counts and offsets.
// With more than kPermPlaceMaxTiles tiles the second step is split in two,
// so that no block reads every tile's counts: perm_scan_kernel (one block)
// turns the counts into totals, offsets and each tile's first position per
// expert, and perm_scatter_kernel places the pairs from those.
// Ids outside [0, E) are skipped: not counted, scatter_indx = -1.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "moe_routing.h"

namespace moe {

int set_error(int status, const char* msg);
int set_cuda_error(cudaError_t err, const char* what);

namespace {

constexpr int kPermTile = 1024;    // pairs per block
constexpr int kPermThreads = 256;  // 8 warps; each warp owns 128 consecutive pairs of the tile
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermMaxE = 1024;
// Up to this many tiles every block of the placing launch sums the tile
// counts itself (tiles x E reads per block, from L2); beyond it a single scan
// block does (three launches).
constexpr int kPermPlaceMaxTiles = 512;
// Dynamic shared memory of the placing launch when it stages the tile counts.
constexpr size_t kPermStageBytes = 192 * 1024;

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__global__ void __launch_bounds__(kPermThreads) perm_count_kernel(const int32_t* __restrict__ ids, int64_t n, int E,
                                                                  int32_t* __restrict__ tile_counts) {
    __shared__ int32_t h[kPermMaxE];
    griddep_launch_dependents();
    for (int e = threadIdx.x; e < E; e += kPermThreads) h[e] = 0;
    __syncthreads();
    // the ids may be written by the previous kernel in the stream
    griddep_wait();
    const int64_t t0 = (int64_t)blockIdx.x * kPermTile;
    constexpr int kPer = kPermTile / kPermThreads;  // pairs per thread, loaded before any is counted
    int idv[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = t0 + threadIdx.x + u * kPermThreads;
        idv[u] = i < n ? __ldg(ids + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u)
        if (idv[u] >= 0 && idv[u] < E) atomicAdd(&h[idv[u]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kPermThreads) tile_counts[(int64_t)blockIdx.x * E + e] = h[e];
}

// 16-byte asynchronous copy global -> shared (through L2), and the wait for
// all of this thread's copies.
__device__ __forceinline__ void cp_async16(int32_t* dst, const int32_t* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 16-byte load through L2 (the tile counts were written by the previous
// kernel); volatile so that a batch of them is issued before any is used.
__device__ __forceinline__ int4 ldcg_v4(const int4* p) {
    int4 v;
    asm volatile("ld.global.cg.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(kPermThreads)
    perm_place_kernel(const int32_t* __restrict__ ids, const float* __restrict__ weights, int64_t n, int E,
                      int ntiles, int stage_counts, const int32_t* __restrict__ tile_counts,
                      int32_t* __restrict__ counts,
                      int32_t* __restrict__ offsets, int32_t* __restrict__ gather, int32_t* __restrict__ scatter,
                      float* __restrict__ gate) {
    extern __shared__ int32_t wbase[];            // [kPermWarps][E]: next position per (warp, expert)
    __shared__ int32_t s_wsum[kPermThreads / 32];
    // [2][ng][E] partial sums of the tile counts (ng * E = 4 * threads), then
    // s_tot (expert totals, then offsets) and s_pre (pairs in earlier tiles)
    __shared__ __align__(16) int32_t s_part[2 * kPermMaxE];
    int32_t* s_tot = s_part;
    int32_t* s_pre = s_part + kPermMaxE;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kRun = kPermTile / kPermWarps;  // pairs per warp
    const int tile = blockIdx.x;
    const int64_t w0 = (int64_t)tile * kPermTile + (int64_t)warp * kRun;
    for (int e = threadIdx.x; e < kPermWarps * E; e += kPermThreads) wbase[e] = 0;
    __syncthreads();
    griddep_wait();  // the tile counts of the first launch
    // this warp's pairs, ids and weights loaded at once, then its counts
    constexpr int kPieces = kRun / 32;
    int idv[kPieces];
    float wv[kPieces];
#pragma unroll
    for (int u = 0; u < kPieces; ++u) {
        const int64_t i = w0 + u * 32 + lane;
        idv[u] = i < n ? __ldg(ids + i) : -1;
        if (idv[u] < 0 || idv[u] >= E) idv[u] = (i < n) ? -2 : -1;  // -2: out of range, -1: past the batch
        wv[u] = (gate != nullptr && idv[u] >= 0) ? __ldg(weights + i) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kPieces; ++u)
        if (idv[u] >= 0) atomicAdd(&wbase[warp * E + idv[u]], 1);
    // Per expert: pairs in earlier tiles (pre) and in all tiles (tot).  The
    // [tiles][E] counts sit in L2; to have many loads in flight, thread
    // (g, c) reads 16-byte column c (4 experts) of every ng-th tile from g,
    // then the ng partial sums meet in shared memory.
    if (stage_counts) {
        // All tile counts into shared memory by asynchronous 16-byte copies
        // (every copy in flight at once, no registers held), then per-expert
        // sums from there.
        int32_t* s_counts = wbase + kPermWarps * E;  // [ntiles][E]
        const int nv = ntiles * E / 4;
        for (int v = threadIdx.x; v < nv; v += kPermThreads) cp_async16(s_counts + 4 * v, tile_counts + 4 * v);
        cp_async_wait_all();
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += kPermThreads) {
            // 8 independent partial sums keep 8 shared-memory loads in flight
            int32_t pre[8] = {0, 0, 0, 0, 0, 0, 0, 0}, tot[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            int j = 0;
            for (; j + 8 <= ntiles; j += 8) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int32_t v = s_counts[(j + u) * E + e];
                    tot[u] += v;
                    pre[u] += (j + u < tile) ? v : 0;
                }
            }
            for (; j < ntiles; ++j) {
                const int32_t v = s_counts[j * E + e];
                tot[0] += v;
                pre[0] += (j < tile) ? v : 0;
            }
            int32_t sp = 0, st = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                sp += pre[u];
                st += tot[u];
            }
            s_pre[e] = sp;
            s_tot[e] = st;
        }
    } else if (E % 4 == 0) {
        const int ncol = E / 4;  // <= 256
        const int ng = kPermThreads / ncol;
        int4 pre = make_int4(0, 0, 0, 0), tot = make_int4(0, 0, 0, 0);
        const int c = threadIdx.x % ncol, g = threadIdx.x / ncol;
        if (g < ng) {
            const int4* col = reinterpret_cast<const int4*>(tile_counts) + c;
            // batches of kBatch loads issued before any is used
            constexpr int kBatch = 16;
            for (int j0 = g; j0 < ntiles; j0 += kBatch * ng) {
                int4 v[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int j = j0 + u * ng;
                    v[u] = make_int4(0, 0, 0, 0);
                    if (j < ntiles) v[u] = ldcg_v4(col + (int64_t)j * ncol);
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int j = j0 + u * ng;
                    tot.x += v[u].x; tot.y += v[u].y; tot.z += v[u].z; tot.w += v[u].w;
                    if (j < tile) {
                        pre.x += v[u].x; pre.y += v[u].y; pre.z += v[u].z; pre.w += v[u].w;
                    }
                }
            }
            reinterpret_cast<int4*>(s_part)[g * ncol + c] = pre;
            reinterpret_cast<int4*>(s_part + 4 * kPermThreads)[g * ncol + c] = tot;
        }
        __syncthreads();
        constexpr int EPT = kPermMaxE / kPermThreads;  // experts per thread, at most
        int32_t sp[EPT], st[EPT];
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
            const int e = threadIdx.x + u * kPermThreads;
            sp[u] = 0;
            st[u] = 0;
            if (e < E) {
                for (int q = 0; q < ng; ++q) {
                    sp[u] += s_part[q * E + e];
                    st[u] += s_part[4 * kPermThreads + q * E + e];
                }
            }
        }
        __syncthreads();  // s_pre and s_tot overlay the partial sums
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
            const int e = threadIdx.x + u * kPermThreads;
            if (e < E) {
                s_pre[e] = sp[u];
                s_tot[e] = st[u];
            }
        }
    } else {
        for (int e = threadIdx.x; e < E; e += kPermThreads) {
            int32_t pre = 0, post = 0;
            int j = 0;
#pragma unroll 8
            for (; j < tile; ++j) pre += __ldcg(tile_counts + (int64_t)j * E + e);
#pragma unroll 8
            for (; j < ntiles; ++j) post += __ldcg(tile_counts + (int64_t)j * E + e);
            s_pre[e] = pre;
            s_tot[e] = pre + post;
        }
    }
    __syncthreads();
    // exclusive scan of the totals over the experts: each thread a contiguous
    // run of experts, then the runs' sums across the block
    const int per = (E + kPermThreads - 1) / kPermThreads;
    const int e0 = threadIdx.x * per, e1 = min(E, e0 + per);
    int32_t run = 0;
    for (int e = e0; e < e1; ++e) run += s_tot[e];
    int32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int32_t wprev = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) {
        const int32_t v = s_wsum[w];
        wprev += w < warp ? v : 0;
        total += v;
    }
    int32_t off = wprev + incl - run;
    for (int e = e0; e < e1; ++e) {
        const int32_t c = s_tot[e];
        if (tile == 0) {
            counts[e] = c;
            offsets[e] = off;
        }
        s_tot[e] = off;
        off += c;
    }
    if (tile == 0 && threadIdx.x == 0) offsets[E] = total;
    __syncthreads();
    // first position of each (warp, expert) of this tile
    for (int e = threadIdx.x; e < E; e += kPermThreads) {
        int32_t r = s_tot[e] + s_pre[e];
        for (int w = 0; w < kPermWarps; ++w) {
            const int32_t c = wbase[w * E + e];
            wbase[w * E + e] = r;
            r += c;
        }
    }
    __syncthreads();
    // place the warp's pairs in order, 32 at a time
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int u = 0; u < kPieces; ++u) {
        const int64_t i = w0 + u * 32 + lane;
        const int id = idv[u] >= 0 ? idv[u] : -1;
        if (idv[u] == -2) scatter[i] = -1;
        const unsigned same = __match_any_sync(0xffffffffu, id);
        int32_t pos = 0;
        if (id >= 0) pos = wbase[warp * E + id] + __popc(same & lt);
        __syncwarp();
        if (id >= 0) {
            gather[pos] = (int32_t)i;
            scatter[i] = pos;
            if (gate) gate[pos] = wv[u];
            if ((same >> lane) == 1u) wbase[warp * E + id] = pos + 1;  // the group's last lane
        }
        __syncwarp();
    }
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
    perm_count_kernel<<<ntiles, kPermThreads, 0, st>>>(topk_ids, n, E, tiles);
    if (ntiles > kPermPlaceMaxTiles || (reinterpret_cast<uintptr_t>(workspace) % 16) != 0) {
        // many tiles: one scan block instead of every block summing all tiles
        // (also for a workspace that 16-byte loads cannot read)
        const int e32 = ((E + 31) / 32) * 32;
        perm_scan_kernel<<<1, e32 * (kPermMaxE / e32), 0, st>>>(tiles, ntiles, E, expert_counts, expert_offsets);
        perm_scatter_kernel<<<ntiles, kPermThreads, sizeof(int32_t) * kPermWarps * E, st>>>(
            topk_ids, topk_weights, n, E, tiles, gather_indx, scatter_indx, gate_scal);
    } else {
        // Stage every tile's counts in shared memory when they fit (with the
        // warps' cursors, at most kPermStageBytes); else sum them from L2.
        const size_t cursors = sizeof(int32_t) * (size_t)kPermWarps * E;
        const size_t staged = sizeof(int32_t) * (size_t)ntiles * E;
        const int stage = (E % 4 == 0 && cursors + staged <= kPermStageBytes) ? 1 : 0;
        const size_t smem = cursors + (stage ? staged : 0);
        if (stage) {  // dynamic + static shared memory may exceed the default 48 KB
            static std::mutex mu;
            static std::unordered_map<int, bool> done;  // device ordinal -> attribute set
            int dev = 0;
            cudaError_t e0 = cudaGetDevice(&dev);
            if (e0 != cudaSuccess) return set_cuda_error(e0, "moe_expert_permutation: cudaGetDevice");
            std::lock_guard<std::mutex> lk(mu);
            if (!done[dev]) {
                e0 = cudaFuncSetAttribute(perm_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kPermStageBytes);
                if (e0 != cudaSuccess) return set_cuda_error(e0, "moe_expert_permutation: kernel attribute");
                done[dev] = true;
            }
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)ntiles, 1, 1);
        cfg.blockDim = dim3((unsigned)kPermThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t err = cudaLaunchKernelEx(&cfg, perm_place_kernel, topk_ids, topk_weights, n, E, ntiles, stage,
                                 static_cast<const int32_t*>(tiles), expert_counts, expert_offsets, gather_indx,
                                 scatter_indx, gate_scal);
        if (err != cudaSuccess) return set_cuda_error(err, "moe_expert_permutation: launch");
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_cuda_error(err, "moe_expert_permutation: launch");
    return MOE_OK;
}

}  // extern "C"
