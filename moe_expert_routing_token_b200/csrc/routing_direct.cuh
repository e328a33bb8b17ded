// Direct routing kernel for topk <= 8 and E = 160 or 256: the SGLang MoE
// routing page's §2-§4 routing ("[SGLang] MoE 라우팅: 토큰에서 전문가로의 배분
// 알고리즘": softmax top-k, grouped top-k, sigmoid + correction_bias with the
// top-2-sum group score), shaped for latency rather than for a ring.
//
// Every warp is its own producer and consumer; no warp waits for another.
//
//  * Staging.  A warp owns "octets" of R = 32 / L token rows, L = 4 or 8
//    lanes per row and C = E / L experts per lane (the library dispatches
//    L = 8 at every batch size).  One elected lane brings an octet into
//    shared memory with bulk asynchronous copies completing on the warp's
//    mbarrier, so the whole octet is in flight with no register cost; a warp
//    keeps kDirectStages octets in flight, and all loads of a call are issued
//    at entry when the grid covers the batch.  For E = 256 (rows of 512 or
//    1024 bytes) one 2-D TMA copy moves the octet, the logits seen as rows of
//    128 bytes with the 128-byte swizzle: a lane's segment is one or two of
//    those rows, and the swizzle spreads the lanes of a row (and the rows
//    of a quarter-warp) over distinct bank groups.  For E = 160 each
//    row is copied to a padded shared-memory row (or the octet in one copy
//    when no padding is needed), which spreads the banks the same way (the
//    library takes that shape for fp32 rows, 20 experts per lane).  The
//    register order of every lane's experts is its segment order.
//  * Threshold.  Each lane scores its C experts (selection keys), takes the
//    maxima of blocks of 8 experts (the first 16 of 20 with E = 160; blocks
//    of a quarter of a group when groups are selected), and the row's L
//    lanes find tau, the k-th largest of each lane's two (L = 8) or four
//    (L = 4) largest block maxima, with a merge network over xor-shuffles:
//    tau is a lower bound for the k-th best key, since the maxima belong to
//    distinct experts.  With group selection the kept groups are ranked
//    first and tau is the k-th largest of their block maxima.
//  * Candidates.  Experts with key >= tau - band (about 10 per row on the
//    benchmark workloads) are appended to a per-row list; the row's L
//    lanes then share the list evenly, compute the exact keys of their
//    entries and rank each one by counting the candidates above it.  The rank
//    is the output slot, so the ids leave in descending key order.  When no
//    row of the warp has more than 16 candidates (nearly always), the list
//    is padded to 16 and ranked in straight-line code: each lane reads the
//    16 keys once for both of its entries.  Exact keys that tie (bf16
//    logits repeat, so a few rows per thousand have them) are detected from
//    the rank sum and ranked again with ties to the lower expert index.  A row with more than kDirectCap
//    candidates or fewer than k (massive ties, NaN scores) is routed by the
//    whole warp: E / 32 exact keys per lane and k rounds of warp arg-max.
//
// Selection keys may approximate the exact keys as long as |phase-1 key -
// exact key| <= eps for every expert: then k experts have exact keys >= tau -
// eps, so every exact top-k expert has a phase-1 key >= tau - 2 eps = tau -
// band and is a candidate.  Key modes:
//  * kKeyRaw: the logit itself (softmax; sigmoid without bias and every group
//    kept).  Both scores are strictly increasing in the logit, so the order is
//    the order of the scores; eps = 0.
//  * kKeyApprox (sigmoid + bias, every group kept): 0.5 tanh(x/2) + (0.5 + b)
//    with the hardware tanh; eps covers kTanhApproxErr and fp32 roundings.
//  * kKeyExact (sigmoid with group selection): the paired-reciprocal sigmoid
//    plus bias for the group scores and the threshold; eps = kPairKeyErr plus
//    roundings.
#pragma once

#include "routing_common.cuh"
#include "routing_threshold.cuh"
#include "sm100_ptx.cuh"

namespace moe {

static __device__ unsigned int g_watchdog_trips_direct;

constexpr int kDirectWarps = 4;
constexpr int kDirectThreads = kDirectWarps * 32;
constexpr int kDirectCap = 32;     // candidates per row on the fast path
constexpr int kDirectFastN = 16;   // list length when every row of the warp has at most this many
constexpr int kDirectStages = 2;   // octets a warp keeps in flight

enum KeyMode : int { kKeyRaw = 0, kKeyApprox = 1, kKeyExact = 2 };

// Bank-conflict check of the row-copy staging layout: for every quarter-warp
// (8 lanes, one 16-byte read each) and every chunk step q, lane l (row l / 4,
// segment l % 4) reads chunk q of its segment at byte r * row_stride + s * seg
// + 16 q, and the 16-byte bias vectors of that chunk at s * bias_stride +
// q * epc * 4 (+16 per further vector); all must fall in distinct 16-byte bank
// groups (equal addresses broadcast).
constexpr bool direct_rows_ok(int row_stride, int seg, int chunks, int epc, int bias_stride) {
    for (int phase = 0; phase < 4; ++phase) {
        for (int q = 0; q < chunks; ++q) {
            unsigned used = 0;
            for (int t = 0; t < 8; ++t) {
                const int l = phase * 8 + t, r = l / 4, s = l % 4;
                const unsigned bit = 1u << (((r * row_stride + s * seg + 16 * q) % 128) / 16);
                if (used & bit) return false;
                used |= bit;
            }
            for (int h = 0; h * 4 < epc; ++h) {
                int addr[8] = {};
                for (int t = 0; t < 8; ++t) {
                    const int l = phase * 8 + t, s = l % 4;
                    addr[t] = s * bias_stride + q * epc * 4 + 16 * h;
                    for (int u = 0; u < t; ++u)
                        if (addr[u] != addr[t] && (addr[u] % 128) / 16 == (addr[t] % 128) / 16) return false;
                }
            }
        }
    }
    return true;
}

// Smallest conflict-free row stride of the row-copy layout (-1 if none).
constexpr int direct_row_stride(int row_bytes, int seg, int chunks, int epc, int bias_stride) {
    for (int pad = 0; pad < 256; pad += 16)
        if (direct_rows_ok(row_bytes + pad, seg, chunks, epc, bias_stride)) return row_bytes + pad;
    return -1;
}

// L lanes per row (4 or 8), R = 32 / L rows per warp pass ("octet").
template <typename TIn, int E, int L_>
struct DirectShape {
    static constexpr int L = L_;
    static constexpr int ESZ = sizeof(TIn);
    static constexpr int C = E / L;                  // experts per lane
    static constexpr int R = 32 / L;                 // rows per octet
    static constexpr int ROW_BYTES = E * ESZ;
    static constexpr int SEG = C * ESZ;              // bytes of a lane's segment
    static constexpr int CH = SEG / 16;              // 16-byte chunks per segment
    static constexpr int EPC = 16 / ESZ;             // experts per chunk
    static constexpr int CQ = (C / 4) | 1;           // padded bias layout: odd float4 count per lane
    static constexpr int CS = CQ * 4;
    // TMA staging: segments of whole 128-byte swizzle rows
    static constexpr bool TMA = E == 256;            // rows of 512 or 1024 bytes: swizzled TMA staging
    static constexpr int TROWS = ROW_BYTES / 128;    // swizzle rows per token row (TMA)
    static constexpr int RS = TMA ? ROW_BYTES : direct_row_stride(ROW_BYTES, SEG, CH, EPC, CS * 4);
    static constexpr int STAGE = R * RS;             // bytes per staged octet (a multiple of 1024 for TMA)
    static constexpr int NB = C / 8;                 // blocks of 8 experts per lane
    static constexpr int MW = (C + 31) / 32;         // candidate mask words per lane
    static_assert((L == 4 || L == 8) && E % L == 0 && SEG % 16 == 0 && C % 4 == 0 && 8 % EPC == 0,
                  "unsupported direct shape");
    static_assert(RS > 0 && RS % 16 == 0, "no conflict-free staging layout");
    static_assert(!TMA || STAGE % 1024 == 0, "swizzled stages start on 1024-byte boundaries");
    static_assert(MW <= 2, "at most 64 experts per lane");
};

// Byte offset, within a staged octet, of chunk q (16 bytes) of lane segment s
// of row r.  TMA staging: the 16-byte chunk c of swizzle row sr sits at
// chunk c ^ (sr mod 8) of that row.
template <typename S>
__device__ __forceinline__ int direct_chunk_off(int r, int s, int q) {
    const int byte = r * S::ROW_BYTES + s * S::SEG + 16 * q;
    if constexpr (S::TMA) {
        const int sr = byte >> 7;
        return (sr << 7) + ((((byte >> 4) & 7) ^ (sr & 7)) << 4);
    } else {
        return r * S::RS + s * S::SEG + 16 * q;
    }
}

// Per-warp candidate lists: R rows of up to kDirectCap entries.  key:
// orderable exact key (0 pads the list), id: the expert; out: the winners by
// output slot, (p, id) with p the unbiased score (sigmoid) or the logit
// (softmax).  Row strides are an odd number of 16-byte vectors (key) or of
// words (id), so that the rows of a warp fall in different banks.
constexpr int kListKeyStride = kDirectCap + 4;  // 36 words: 9 vectors
constexpr int kListStride = kDirectCap + 1;     // 33 words
template <int R>
struct DirectLists {
    uint32_t key[R][kListKeyStride];
    int id[R][kListStride];
    float2 out[R][9];  // by output slot: (p, id) of the winner
};

template <typename TIn, int E, int L>
constexpr size_t direct_smem_bytes() {
    using S = DirectShape<TIn, E, L>;
    return 1024 + (size_t)kDirectWarps * kDirectStages * S::STAGE +     // staged octets
           (size_t)kDirectWarps * sizeof(DirectLists<S::R>) +          // candidate lists
           (size_t)S::L * S::CS * 4 + (size_t)E * 4 +                  // bias tables
           (size_t)kDirectWarps * kDirectStages * 8 +                  // mbarriers
           (size_t)kDirectWarps * 4;                                   // per-warp max |bias|
}

// Compare-exchange, descending.
__device__ __forceinline__ void dcx(float& a, float& b) {
    const float hi = fmaxf(a, b);
    b = fminf(a, b);
    a = hi;
}

template <int N>
__device__ __forceinline__ void sort_desc(float (&v)[N]) {
    static_assert(N == 4 || N == 8, "sorting network for 4 or 8 values");
    if constexpr (N == 4) {
        dcx(v[0], v[1]); dcx(v[2], v[3]); dcx(v[0], v[2]); dcx(v[1], v[3]); dcx(v[1], v[2]);
    } else {  // Batcher's odd-even merge sort, 19 compare-exchanges
        dcx(v[0], v[1]); dcx(v[2], v[3]); dcx(v[4], v[5]); dcx(v[6], v[7]);
        dcx(v[0], v[2]); dcx(v[1], v[3]); dcx(v[4], v[6]); dcx(v[5], v[7]);
        dcx(v[1], v[2]); dcx(v[5], v[6]);
        dcx(v[0], v[4]); dcx(v[1], v[5]); dcx(v[2], v[6]); dcx(v[3], v[7]);
        dcx(v[2], v[4]); dcx(v[3], v[5]);
        dcx(v[1], v[2]); dcx(v[3], v[4]); dcx(v[5], v[6]);
    }
}

// The K-th largest (1 <= K <= 8) and the largest of the L * P values held P
// per lane by the L lanes of a row (P = 4 or 8, any order; -inf pads).  Sort
// locally, then log2(L) xor-shuffle rounds each merge two sorted lists:
// concatenation while the result fits in 8, else the top 8 of the two
// (elementwise max against the reversed partner, a bitonic sequence).  For
// K = 8 the last round needs only the minimum of that top 8.
template <int P, int L>
__device__ __forceinline__ float row_kth(const float (&in)[P], int K, float& vmax) {
    float a[8];
    {
        float s[P];
#pragma unroll
        for (int i = 0; i < P; ++i) s[i] = in[i];
        sort_desc(s);
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = i < P ? s[i] : -INFINITY;
    }
    if constexpr (P == 4) {  // two sorted 4-lists -> one sorted 8-list
#pragma unroll
        for (int i = 0; i < 4; ++i) a[7 - i] = __shfl_xor_sync(kFullMask, a[i], 1);
        bitonic_clean_desc(a);
    } else {  // top 8 of two sorted 8-lists
        float b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = __shfl_xor_sync(kFullMask, a[i], 1);
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fmaxf(a[i], b[7 - i]);
        bitonic_clean_desc(a);
    }
#pragma unroll
    for (int o = 2; o < L; o <<= 1) {
        float b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = __shfl_xor_sync(kFullMask, a[i], o);
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fmaxf(a[i], b[7 - i]);
        if ((o << 1) < L) bitonic_clean_desc(a);
    }
    if (K == 8) {
        vmax = fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
        return fminf(fminf(fminf(a[0], a[1]), fminf(a[2], a[3])), fminf(fminf(a[4], a[5]), fminf(a[6], a[7])));
    }
    bitonic_clean_desc(a);
    vmax = a[0];
    return kth_of_sorted8(a, K);
}

// Unpack one 16-byte chunk into fp32 values.
template <typename TIn>
__device__ __forceinline__ void unpack_chunk(const uint4& v, float* x);
template <>
__device__ __forceinline__ void unpack_chunk<__nv_bfloat16>(const uint4& v, float* x) {
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x); x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z); x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}
template <>
__device__ __forceinline__ void unpack_chunk<float>(const uint4& v, float* x) {
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y); x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
}

// Half of each bf16 value of a packed pair (a bf16 multiply by 0.5, exact
// unless the result is subnormal).
__device__ __forceinline__ uint32_t bf16x2_half(uint32_t w) {
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0x3F003F00u), "r"(0x80008000u));
    return r;
}

template <typename TIn>
__device__ __forceinline__ float staged_logit(const uint8_t* seg, int i) {
    if constexpr (sizeof(TIn) == 2)
        return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(seg + 2 * i)) << 16);
    else
        return *reinterpret_cast<const float*>(seg + 4 * i);
}

// The exact selection key and unbiased score of one expert from its logit.
template <int SCORE, bool BIAS, int MODE>
__device__ __forceinline__ void exact_key(float x, float b, float& key, float& p) {
    if constexpr (SCORE == kSoftmax) {
        key = x;
        p = x;
    } else {
        p = sigmoid_f32(x);
        if constexpr (MODE == kKeyRaw) key = x;  // sigmoid without bias: the logit orders the scores
        else key = BIAS ? p + b : p;
    }
}

// GS: experts per group when groups are selected (the lane owns C / GS whole
// groups), 0 when every group is kept.
// Resident blocks per SM the compiler is asked to fit, the most that compile
// without spills.  Eight lanes per bf16 row: 8 (64 registers) for
// approximate keys, 7 (72) for the other sigmoid keys, 5 (96) for softmax;
// at 16384 rows that puts (nearly) one octet per warp in flight.  fp32
// E = 160: 5 (96).  Other shapes: 4 (128 registers).
template <typename TIn, int E, int L, int SCORE, int MODE>
constexpr int direct_min_blocks() {
    if (L != 8) return 4;
    if (sizeof(TIn) != 2) return E == 160 ? 5 : 4;
    return SCORE == kSoftmax ? 5 : (MODE == kKeyApprox ? 8 : 7);
}

template <typename TIn, int E, int L_, int SCORE, bool BIAS, int MODE, int GS>
__global__ void __launch_bounds__(kDirectThreads, direct_min_blocks<TIn, E, L_, SCORE, MODE>())
    route_direct_kernel(const __grid_constant__ CUtensorMap tmap, RouteArgs a, int64_t n_oct) {
    using S = DirectShape<TIn, E, L_>;
    constexpr int C = S::C, R = S::R, L = S::L, D = kDirectStages, EPC = S::EPC, CH = S::CH;
    constexpr bool GROUPED = GS > 0;
    constexpr int NG = GROUPED ? C / GS : 1;  // groups per lane
    static_assert(!GROUPED || (C % (GS > 0 ? GS : 1) == 0 && NG <= 4), "a lane owns whole groups");
    static_assert(MODE != kKeyApprox || (SCORE == kSigmoid && !GROUPED), "approximate keys: sigmoid, all groups");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = ptx::smem_align<1024>(smem_raw);
    uint8_t* stages = base;
    DirectLists<R>* lists = reinterpret_cast<DirectLists<R>*>(stages + (size_t)kDirectWarps * D * S::STAGE);
    float* s_b1 = reinterpret_cast<float*>(lists + kDirectWarps);  // phase-1 key offsets, padded lane layout
    float* s_b2 = s_b1 + L * S::CS;                                // exact bias by expert
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_b2 + E);
    float* s_bmax = reinterpret_cast<float*>(bars + kDirectWarps * D);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int sl = lane % L;      // segment (lane) within the row
    const int rr = lane / L;      // row within the octet
    const int seg0 = rr * L;      // first lane of this row's segment
    uint8_t* my_stages = stages + (size_t)warp * D * S::STAGE;
    uint64_t* my_bars = bars + warp * D;
    DirectLists<R>& lst = lists[warp];
    const int64_t nwarps = (int64_t)gridDim.x * kDirectWarps;
    const int64_t gw = (int64_t)blockIdx.x * kDirectWarps + warp;


    if (lane == 0) {
#pragma unroll
        for (int d = 0; d < D; ++d) ptx::mbar_init(&my_bars[d], 1);
        ptx::fence_mbar_init();
        if constexpr (S::TMA) ptx::tma_prefetch_desc(&tmap);
    }
    __syncwarp();
    // Inputs may be written by the previous kernel in the stream: wait for it.
    ptx::griddep_wait();

    const uint8_t* logits = static_cast<const uint8_t*>(a.logits);
    const uint64_t policy = ptx::l2_policy_evict_first();
    auto issue = [&](int64_t oct, int d) {  // lane 0 only
        uint64_t* bar = &my_bars[d];
        uint8_t* dst = my_stages + (size_t)d * S::STAGE;
        if constexpr (S::TMA) {
            // one box of R * TROWS swizzle rows; rows past the tensor are
            // zero-filled and still counted
            ptx::mbar_arrive_expect_tx(bar, (uint32_t)S::STAGE);
            ptx::tma_load_2d(dst, &tmap, 0, (int)(oct * R * S::TROWS), bar, policy);
        } else {
            const int64_t left = a.M - oct * R;
            const int nrows = left < R ? (int)left : R;
            const uint8_t* src = logits + (size_t)(oct * R) * S::ROW_BYTES;
            ptx::mbar_arrive_expect_tx(bar, (uint32_t)(nrows * S::ROW_BYTES));
            if constexpr (S::RS == S::ROW_BYTES) {
                ptx::bulk_g2s(dst, src, (uint32_t)(nrows * S::ROW_BYTES), bar);
            } else {
                for (int r = 0; r < nrows; ++r)
                    ptx::bulk_g2s(dst + r * S::RS, src + (size_t)r * S::ROW_BYTES, S::ROW_BYTES, bar);
            }
        }
    };
    if (lane == 0) {
#pragma unroll
        for (int d = 0; d < D; ++d)
            if (gw + d * nwarps < n_oct) issue(gw + d * nwarps, d);
    }

    // Bias tables and the candidate band: the block's threads share the
    // entries (E / 128 each) and the per-warp maxima of |b| meet in shared
    // memory.
    float bmax = 0.0f;
#pragma unroll
    for (int e0 = 0; e0 < E; e0 += kDirectThreads) {
        const int e = e0 + (int)threadIdx.x;
        if (e < E) {
            const float b = BIAS ? bias_as_used(__ldg(a.bias + e), a.bias_bf16) : 0.0f;
            bmax = fmaxf(bmax, fabsf(b));
            s_b2[e] = b;
            s_b1[(e / C) * S::CS + e % C] = (MODE == kKeyApprox) ? 0.5f + b : b;
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFullMask, bmax, o));
    if (lane == 0) s_bmax[warp] = bmax;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kDirectWarps; ++w) bmax = fmaxf(bmax, s_bmax[w]);
    float band = 0.0f;
    if constexpr (MODE != kKeyRaw) {
        // eps = key error (tanh bound or pair/single difference) + 4 ulp of
        // keys up to 2 + max|b|; band = 2 eps
        const float round = (bmax + 2.0f) * (1.0f / 2097152.0f);
        band = (MODE == kKeyApprox) ? 2.0f * (0.5f * kTanhApproxErr + round) : 2.0f * (kPairKeyErr + round);
    }

    const int K = a.K;
    const float* b1 = s_b1 + sl * S::CS;
    for (int j = 0;; ++j) {
        const int64_t oct = gw + (int64_t)j * nwarps;
        if (oct >= n_oct) break;
        const int d = j % D;
        if (!ptx::mbar_wait(&my_bars[d], (uint32_t)((j / D) & 1), kWaitBudgetNs)) {
            // The copies did not land in time: count it, wait (bounded) for the
            // copies this warp still has in flight, and stop.
            if (lane == 0) atomicAdd(&g_watchdog_trips_direct, 1u);
            for (int k = 1; k < D; ++k) {
                const int jj = j + k;
                if (gw + (int64_t)jj * nwarps < n_oct)
                    ptx::mbar_wait(&my_bars[jj % D], (uint32_t)((jj / D) & 1), kWaitBudgetNs);
            }
            return;
        }
        const uint8_t* stage = my_stages + (size_t)d * S::STAGE;
        // logit of lane-local expert li of segment s_ of this lane's row
        auto logit_at = [&](int s_, int li) {
            return staged_logit<TIn>(stage + direct_chunk_off<S>(rr, s_, li / EPC), li % EPC);
        };
        const int64_t row = oct * R + rr;
        const bool valid = row < a.M;

        // ---- keys -----------------------------------------------------------
        float key[C];
#pragma unroll
        for (int q = 0; q < CH; ++q) {
            const int c = q;
            const uint4 v = *reinterpret_cast<const uint4*>(stage + direct_chunk_off<S>(rr, sl, q));
            if constexpr (MODE == kKeyApprox) {
                float h[EPC];
                if constexpr (sizeof(TIn) == 2) {
                    const uint4 hv = make_uint4(bf16x2_half(v.x), bf16x2_half(v.y), bf16x2_half(v.z), bf16x2_half(v.w));
                    unpack_chunk<TIn>(hv, h);
                } else {
                    unpack_chunk<TIn>(v, h);
#pragma unroll
                    for (int i = 0; i < EPC; ++i) h[i] *= 0.5f;
                }
#pragma unroll
                for (int u = 0; u < EPC / 4; ++u) {
                    const float4 b = reinterpret_cast<const float4*>(b1 + c * EPC)[u];
                    key[q * EPC + 4 * u + 0] = fmaf(tanh_approx(h[4 * u + 0]), 0.5f, b.x);
                    key[q * EPC + 4 * u + 1] = fmaf(tanh_approx(h[4 * u + 1]), 0.5f, b.y);
                    key[q * EPC + 4 * u + 2] = fmaf(tanh_approx(h[4 * u + 2]), 0.5f, b.z);
                    key[q * EPC + 4 * u + 3] = fmaf(tanh_approx(h[4 * u + 3]), 0.5f, b.w);
                }
            } else {
                float x[EPC];
                unpack_chunk<TIn>(v, x);
                if constexpr (MODE == kKeyExact) {
#pragma unroll
                    for (int u = 0; u < EPC / 4; ++u) {
                        const float4 b = reinterpret_cast<const float4*>(b1 + c * EPC)[u];
                        const unsigned long long k01 =
                            sigmoid_pair(pack2(fmaxf(x[4 * u], kSigmoidClamp), fmaxf(x[4 * u + 1], kSigmoidClamp)));
                        const unsigned long long k23 = sigmoid_pair(
                            pack2(fmaxf(x[4 * u + 2], kSigmoidClamp), fmaxf(x[4 * u + 3], kSigmoidClamp)));
                        key[q * EPC + 4 * u + 0] = lo2(k01) + b.x;
                        key[q * EPC + 4 * u + 1] = hi2(k01) + b.y;
                        key[q * EPC + 4 * u + 2] = lo2(k23) + b.z;
                        key[q * EPC + 4 * u + 3] = hi2(k23) + b.w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < EPC; ++i) key[q * EPC + i] = x[i];
                }
            }
        }

        // ---- kept groups and threshold --------------------------------------
        float tau, rowmax;
        uint32_t keep_bits[S::MW];  // admissible register slots of this lane
#pragma unroll
        for (int w = 0; w < S::MW; ++w) keep_bits[w] = (w * 32 + 32 <= C) ? 0xffffffffu : ((1u << (C % 32)) - 1u);
        if constexpr (GROUPED) {
            // top-2 of each local group
            float m1[NG], m2[NG];
#pragma unroll
            for (int u = 0; u < NG; ++u) {
                m1[u] = -INFINITY;
                m2[u] = -INFINITY;
            }
#pragma unroll
            for (int i = 0; i < C; ++i) {
                top2_push(m1[i / GS], m2[i / GS], key[i]);
            }
            float gsc[NG];
#pragma unroll
            for (int u = 0; u < NG; ++u) gsc[u] = (a.group_kind == kGroupTop2Sum && GS > 1) ? m1[u] + m2[u] : m1[u];
            // rank every local group against all groups of the row (ties to
            // the lower group index)
            int rank[NG];
#pragma unroll
            for (int u = 0; u < NG; ++u) rank[u] = 0;
#pragma unroll
            for (int jl = 0; jl < L; ++jl) {
#pragma unroll
                for (int v = 0; v < NG; ++v) {
                    const float o = __shfl_sync(kFullMask, gsc[v], seg0 + jl);
                    const int og = jl * NG + v;
#pragma unroll
                    for (int u = 0; u < NG; ++u) rank[u] += (o > gsc[u]) || (o == gsc[u] && og < sl * NG + u);
                }
            }
            static_assert(NG <= 2, "at most two groups per lane");
            constexpr int BSZ = GS / 4;  // four blocks per group
            float mx = -INFINITY;
#pragma unroll
            for (int u = 0; u < NG; ++u) mx = fmaxf(mx, m1[u]);
            bool kept[NG];
            float tv[4];
            {
                float bm[8];
#pragma unroll
                for (int u = 0; u < NG; ++u) {
                    kept[u] = rank[u] < a.TG;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        float m = -INFINITY;
#pragma unroll
                        for (int i = 0; i < BSZ; ++i) m = fmaxf(m, key[u * GS + b * BSZ + i]);
                        bm[4 * u + b] = kept[u] ? m : -INFINITY;
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) tv[i] = bm[i];
                if constexpr (NG == 2) {
                    float h[4] = {bm[4], bm[5], bm[6], bm[7]};
                    sort_desc(tv);
                    sort_desc(h);
#pragma unroll
                    for (int i = 0; i < 4; ++i) tv[i] = fmaxf(tv[i], h[3 - i]);
                }
            }
            // experts of dropped groups are not admissible
#pragma unroll
            for (int i = 0; i < C; ++i)
                if (!kept[i / GS]) keep_bits[i / 32] &= ~(1u << (i % 32));
            // the k-th largest of the kept groups' block maxima (distinct
            // experts: a lower bound for the k-th best admissible key)
            float dummy;
            tau = row_kth<4, L>(tv, K, dummy);
            rowmax = mx;
#pragma unroll
            for (int o = 1; o < L; o <<= 1) rowmax = fmaxf(rowmax, __shfl_xor_sync(kFullMask, rowmax, o));
        } else {
            float bm[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) bm[i] = -INFINITY;
#pragma unroll
            for (int u = 0; u < S::NB; ++u) {
                const float* k8 = key + 8 * u;
                bm[u] = fmax3(fmax3(k8[0], k8[1], k8[2]), fmax3(k8[3], k8[4], k8[5]), fmaxf(k8[6], k8[7]));
            }
            if constexpr (L == 8 && S::NB == 4) {
                // Eight lanes: each contributes its two largest block maxima
                // (16 distinct experts per row, so their k-th largest is a
                // lower bound).
                const float ah = fmaxf(bm[0], bm[1]), al = fminf(bm[0], bm[1]);
                const float ch = fmaxf(bm[2], bm[3]), cl = fminf(bm[2], bm[3]);
                tau = row_kth2<L>(fmaxf(ah, ch), fmax3(fminf(ah, ch), al, cl), K, rowmax);
            } else {
                // Each lane contributes its four largest block maxima: two
                // sorted halves, then the top four of the two.
                float b4[4] = {bm[0], bm[1], bm[2], bm[3]};
                if constexpr (S::NB > 4) {
                    float h[4] = {bm[4], bm[5], bm[6], bm[7]};
                    sort_desc(b4);
                    sort_desc(h);
#pragma unroll
                    for (int i = 0; i < 4; ++i) b4[i] = fmaxf(b4[i], h[3 - i]);
                }
                tau = row_kth<4, L>(b4, K, rowmax);
            }
        }
        const float lo = tau - band;

        // ---- candidate mask: key >= lo, from the sign bits of key - lo ------
        uint32_t cmask[S::MW];
#pragma unroll
        for (int w = 0; w < S::MW; ++w) {
            uint32_t below = 0u;
#pragma unroll
            for (int i = 31; i >= 0; --i) {
                const int e = w * 32 + i;
                if (e < C) {
                    // shift in the sign of key - lo (set: below the band)
                    const float dv = key[e] - lo;
                    asm("shf.l.clamp.b32 %0, %1, %0, 1;" : "+r"(below) : "r"(__float_as_uint(dv)));
                } else {
                    below <<= 1;
                }
            }
            cmask[w] = valid ? (~below & keep_bits[w]) : 0u;
        }
        int cnt = 0;
#pragma unroll
        for (int w = 0; w < S::MW; ++w) cnt += __popc(cmask[w]);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < L; o <<= 1) {
            const int t = __shfl_up_sync(kFullMask, incl, o, L);
            if (sl >= o) incl += t;
        }
        const int n = __shfl_sync(kFullMask, incl, seg0 + L - 1);
        bool slow = valid && (n > kDirectCap || n < K);

        // ---- candidate list: ids first, then exact keys by list position ----
        // Each lane appends its candidates' ids; then the row's L lanes take
        // the list entries t = sl, sl + L, ... (an even share, whatever lane the
        // experts live in), compute their exact keys and rank them.
        if (!slow) {
            int pos = incl - cnt;
#pragma unroll
            for (int w = 0; w < S::MW; ++w) {
                uint32_t bits = cmask[w];
                while (bits) {
                    const int i = w * 32 + __ffs(bits) - 1;
                    bits &= bits - 1u;
                    lst.id[rr][pos++] = sl * C + i;
                }
            }
        }
        const int nf = (valid && !slow) ? n : 0;
        const int nmax = __reduce_max_sync(kFullMask, nf);
        __syncwarp();
        constexpr int TPL = kDirectCap / L;  // list entries per lane
        uint32_t kt[TPL];
        float pt[TPL];
        int it[TPL];
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
            kt[u] = 0u;
            pt[u] = 0.0f;
            it[u] = 0;
        }
        // exact key of list entry t = sl + u * L (0 beyond the row's list)
        auto entry_key = [&](int u) {
            const int t = sl + u * L;
            if (t < nf) {
                const int e = lst.id[rr][t];
                float kx, px;
                exact_key<SCORE, BIAS, MODE>(logit_at(e / C, e % C), BIAS ? s_b2[e] : 0.0f, kx, px);
                kt[u] = order_u32(kx);
                pt[u] = px;
                it[u] = e;
            }
        };
        // ---- rank by counting: slot of candidate t = #candidates above it ---
        // set.gt gives -1 per key above; three-input adds sum them.  The
        // winners (rank < K) go to the row's slot table.
        auto count_above = [](const uint4& k4, uint32_t k0, int c) {
            uint32_t s0, s1, s2, s3;
            asm("set.gt.u32.u32 %0, %1, %2;" : "=r"(s0) : "r"(k4.x), "r"(k0));
            asm("set.gt.u32.u32 %0, %1, %2;" : "=r"(s1) : "r"(k4.y), "r"(k0));
            asm("set.gt.u32.u32 %0, %1, %2;" : "=r"(s2) : "r"(k4.z), "r"(k0));
            asm("set.gt.u32.u32 %0, %1, %2;" : "=r"(s3) : "r"(k4.w), "r"(k0));
            c = c - (int)s0 - (int)s1;
            return c - (int)s2 - (int)s3;
        };
        int rsum = 0;
        if (L == 8 && nmax <= kDirectFastN) {
            // Every row of the warp has at most 16 candidates (nearly all
            // octets): the list is padded to 16 with zero keys, each lane
            // keys 16 / L entries, then reads the 16 keys once and ranks its
            // entries against them.
            constexpr int FS = kDirectFastN / L;
#pragma unroll
            for (int u = 0; u < FS; ++u) {
                entry_key(u);
                lst.key[rr][sl + u * L] = kt[u];
            }
            __syncwarp();
            uint4 k4[kDirectFastN / 4];
#pragma unroll
            for (int q = 0; q < kDirectFastN / 4; ++q) k4[q] = *reinterpret_cast<const uint4*>(&lst.key[rr][4 * q]);
#pragma unroll
            for (int u = 0; u < FS; ++u) {
                const int t = sl + u * L;
                const uint32_t k0 = t < nf ? kt[u] : 0xffffffffu;
                int c = 0;
#pragma unroll
                for (int q = 0; q < kDirectFastN / 4; ++q) c = count_above(k4[q], k0, c);
                if (t < nf) {
                    rsum += c;
                    if (c < K) lst.out[rr][c] = make_float2(pt[u], __int_as_float(it[u]));
                }
            }
        } else {
            const int jmax = (nmax + 3) & ~3;
#pragma unroll
            for (int u = 0; u < TPL; ++u) {
                const int t = sl + u * L;
                if (u * L < nmax) {  // warp-uniform bound
                    entry_key(u);
                    if (t < jmax) lst.key[rr][t] = kt[u];  // 0 pads the list to jmax
                }
            }
            __syncwarp();
#pragma unroll
            for (int u = 0; u < TPL; ++u) {
                if (u * L < nmax) {  // warp-uniform bound
                    const int t = sl + u * L;
                    const uint32_t k0 = t < nf ? kt[u] : 0xffffffffu;
                    int c = 0;
#pragma unroll
                    for (int j4 = 0; j4 < kDirectCap; j4 += 4)
                        if (j4 < jmax) c = count_above(*reinterpret_cast<const uint4*>(&lst.key[rr][j4]), k0, c);
                    if (t < nf) {
                        rsum += c;
                        if (c < K) lst.out[rr][c] = make_float2(pt[u], __int_as_float(it[u]));
                    }
                }
            }
        }
#pragma unroll
        for (int o = 1; o < L; o <<= 1) rsum += __shfl_xor_sync(kFullMask, rsum, o);
        // Distinct keys give ranks 0 .. n-1 (sum n(n-1)/2); equal keys share a
        // rank and lower the sum.  Such rows are ranked again, an equal key
        // with a lower expert index counting as above.
        const bool ties = valid && !slow && rsum != n * (n - 1) / 2;
        if (__any_sync(kFullMask, ties)) {
            __syncwarp();  // the first ranking's slot writes land before these
#pragma unroll
            for (int u = 0; u < TPL; ++u) {
                const int t = sl + u * L;
                if (u * L < nmax) {
                    int c = 0;
                    for (int jj = 0; jj < nf; ++jj) {
                        const uint32_t kj = lst.key[rr][jj];
                        c += (kj > kt[u]) || (kj == kt[u] && lst.id[rr][jj] < it[u]);
                    }
                    if (ties && t < nf && c < K) lst.out[rr][c] = make_float2(pt[u], __int_as_float(it[u]));
                }
            }
        }

        // ---- rare rows: the whole warp routes each one by k exact rounds of
        // arg-max (E / 32 experts per lane), ties to the lower index ----------
        const unsigned slow_rows = __ballot_sync(kFullMask, slow && sl == 0);
        if (slow_rows) {
            __syncwarp();
            constexpr int EPL = E / 32;  // experts per lane
            uint32_t kept_groups = 0xffffffffu;  // of this lane's row, bit g = group g kept
            if constexpr (GROUPED) {
                uint32_t own = 0u;
#pragma unroll
                for (int u = 0; u < NG; ++u) own |= (keep_bits[(u * GS) / 32] >> ((u * GS) % 32) & 1u) << (sl * NG + u);
#pragma unroll
                for (int o = 1; o < L; o <<= 1) own |= __shfl_xor_sync(kFullMask, own, o);
                kept_groups = own;
            }
            unsigned left = slow_rows;
            while (left) {
                const int src = __ffs(left) - 1;
                left &= left - 1u;
                const int r = src / L;
                const uint32_t km = __shfl_sync(kFullMask, kept_groups, src);
                auto logit_re = [&](int e) {
                    const int li = e % C;
                    return staged_logit<TIn>(stage + direct_chunk_off<S>(r, e / C, li / EPC), li % EPC);
                };
                uint32_t ku[EPL];
#pragma unroll
                for (int j = 0; j < EPL; ++j) {
                    const int e = lane * EPL + j;
                    float kx, px;
                    exact_key<SCORE, BIAS, MODE>(logit_re(e), BIAS ? s_b2[e] : 0.0f, kx, px);
                    const bool adm = GROUPED ? ((km >> (e / (GROUPED ? GS : 1))) & 1u) != 0u : true;
                    ku[j] = adm ? order_u32(kx) : 0u;
                }
#pragma unroll 1
                for (int jr = 0; jr < K; ++jr) {
                    uint32_t bk = 0u;
                    int be = 0x7fffffff;
#pragma unroll
                    for (int j = 0; j < EPL; ++j) {
                        const bool better = ku[j] > bk;  // ascending index: ties keep the lower
                        be = better ? lane * EPL + j : be;
                        bk = better ? ku[j] : bk;
                    }
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) {
                        const uint32_t ok = __shfl_xor_sync(kFullMask, bk, o);
                        const int oe = __shfl_xor_sync(kFullMask, be, o);
                        if (ok > bk || (ok == bk && oe < be)) {
                            bk = ok;
                            be = oe;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < EPL; ++j)
                        if (lane * EPL + j == be) ku[j] = 0u;
                    if (lane == 0) {
                        const int eo = (be >= 0 && be < E) ? be : 0;
                        float kx, px;
                        exact_key<SCORE, BIAS, MODE>(logit_re(eo), 0.0f, kx, px);
                        lst.out[r][jr] = make_float2(px, __int_as_float(eo));
                    }
                }
            }
        }
        __syncwarp();

        // ---- weights: gather from the slot table, renormalise, scale, store --
        // Lane sl takes output slot sl (and sl + L, ...): the sum runs over the
        // slots in a fixed order, so a row's weights depend on that row alone.
        float denom_all = 1.0f;
        if constexpr (SCORE == kSoftmax) {
            if (!a.renorm) {
                float s = 0.0f;
#pragma unroll
                for (int i = 0; i < C; ++i) s += softmax_num(key[i], rowmax, a.softcap);  // key = logit
#pragma unroll
                for (int o = 1; o < L; o <<= 1) s += __shfl_xor_sync(kFullMask, s, o);
                denom_all = s;
            }
        }
        auto weight_of = [&](float p) { return (SCORE == kSoftmax) ? softmax_num(p, rowmax, a.softcap) : p; };
        auto scale_of = [&](float wsum) {
#pragma unroll
            for (int o = 1; o < L; o <<= 1) wsum += __shfl_xor_sync(kFullMask, wsum, o);
            if (a.renorm) return __fdividef(a.rsf, wsum);
            return (SCORE == kSoftmax) ? __fdividef(a.rsf, denom_all) : a.rsf;
        };
        {
            constexpr int SPL = (8 + L - 1) / L;  // output slots per lane
            float wv[SPL];
            int iv[SPL];
            float wsum = 0.0f;
#pragma unroll
            for (int v = 0; v < SPL; ++v) {
                const int js = sl + v * L;
                wv[v] = 0.0f;
                iv[v] = 0;
                if (js < K) {
                    const float2 o = lst.out[rr][js];
                    wv[v] = weight_of(o.x);
                    iv[v] = __float_as_int(o.y);
                    wsum += wv[v];
                }
            }
            const float scale = scale_of(wsum);
            if (valid) {
#pragma unroll
                for (int v = 0; v < SPL; ++v) {
                    const int js = sl + v * L;
                    if (js < K) {
                        a.weights[row * K + js] = wv[v] * scale;
                        a.ids[row * K + js] = iv[v];
                    }
                }
            }
        }
        __syncwarp();

        const int64_t next = gw + (int64_t)(j + D) * nwarps;
        if (lane == 0 && next < n_oct) issue(next, d);
    }
    // The next kernel in the stream launches once every warp is done: its
    // blocks would otherwise wait on these SMs and take issue slots.
    ptx::griddep_launch_dependents();
}

}  // namespace moe
