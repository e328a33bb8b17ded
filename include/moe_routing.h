/*
 * moe_routing.h - C ABI of the B200 (sm_100a) Mixture-of-Experts
 * token-to-expert routing library (libmoe_routing.so).
 *
 * Every entry point routes M token rows of router logits to k experts each and
 * writes, per row, k expert ids (int32) and k routing weights (fp32):
 *
 *   scores      softmax over the row, or sigmoid per expert
 *   choice      selection score = score + correction_bias (bias optional)
 *   groups      the E experts form num_expert_group contiguous groups of
 *               S = E / num_expert_group; each group gets a score (its largest
 *               selection score, or the sum of its two largest); the
 *               topk_group best groups are kept and every expert of the other
 *               groups is excluded
 *   top-k       the k best selection scores among the kept experts
 *   weights     the UNBIASED scores of the chosen experts; if renormalize,
 *               divided by their sum; then multiplied by routed_scaling_factor
 *
 * Sources (pages on SGLang MoE routing, cited by title and section):
 *   [R] "[SGLang] MoE 라우팅: 토큰에서 전문가로의 배분 알고리즘"
 *       §2 기본 softmax Top-K, §3 Grouped Top-K, §4 Biased Grouped Top-K,
 *       §5 Fused MoE Router; the fused_topk / grouped_topk_gpu /
 *       biased_grouped_topk_impl signatures shown there
 *   [A] "[sglang] SGLang MoE 라우팅 최적화: AMD GPU에서 aiter.biased_grouped_topk 활용",
 *       코드 분석 (After): the aiter_biased_grouped_topk call with
 *       num_expert_group=1, topk_group=1, need_renorm=renormalize
 *
 * Conventions shared by every call
 *   - Tie-break: between equal selection scores (and equal group scores) the
 *     lower index wins.  Ids are written in descending selection score, ties in
 *     ascending index.  (The pages leave this open; this is the reading taken.)
 *   - Layout: every matrix is row-major and densely packed (row stride = number
 *     of columns).  Outputs are (M, topk) row-major.
 *   - Memory: all pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees, synchronises or prints.  Calls are asynchronous
 *     on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 *     stream) and may be captured in a CUDA graph.
 *   - Errors: the return value is a moe_status_t.  Invalid arguments are
 *     rejected before anything is launched (MOE_ERR_INVALID_ARG); shapes the
 *     library was not built for give MOE_ERR_UNSUPPORTED; a failed launch gives
 *     MOE_ERR_CUDA.  moe_last_error() returns a message for the calling thread's
 *     last failure.  M == 0 is valid and launches nothing.
 *   - Inputs must be finite; NaN or infinity in the logits is outside the
 *     contract (no per-element check is made; the output is then unspecified
 *     but every written id is still in [0, E)).
 *   - Arithmetic is fp32 on the device from bf16 or fp32 inputs.
 */
#ifndef MOE_ROUTING_H
#define MOE_ROUTING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 1: the routing calls and the fused router.  2: adds the allocation-free
 * fused router, the softcap and aiter variants, the expert permutation, the
 * shared-expert slot, the ascending-id order and the bounded-wait self-test
 * (every version-1 call keeps its signature and meaning).  3: adds the
 * small-E top-1 router moe_fused_router_top1 (earlier calls unchanged).  4:
 * adds moe_fill_shared_expert_slot_philox, the shared-expert slot with the
 * library drawing the shared expert from a seed (earlier calls unchanged).
 * 5: moe_fused_router_top1 takes E up to 256 (its tensor-core kernel);
 * calls that version 4 accepted still succeed; with (E, K) weights and
 * K % 64 == 0 they run on the tensor-core kernel, whose fp32 sums are
 * ordered differently. */
#define MOE_ROUTING_ABI_VERSION 5

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* argument outside the documented domain     */
    MOE_ERR_UNSUPPORTED = 2, /* valid, but the library has no kernel for it */
    MOE_ERR_CUDA = 3         /* the CUDA runtime reported an error         */
} moe_status_t;

typedef enum {
    MOE_DTYPE_F32 = 0,
    MOE_DTYPE_BF16 = 1
} moe_dtype_t;

typedef enum {
    MOE_WEIGHT_K_BY_E = 0, /* router weight stored (K, E): hidden x W        */
    MOE_WEIGHT_E_BY_K = 1  /* router weight stored (E, K): nn.Linear layout  */
} moe_weight_layout_t;

/* Library ABI version (MOE_ROUTING_ABI_VERSION of the build). */
MOE_API int moe_abi_version(void);

/* Static text for a status code. */
MOE_API const char* moe_status_string(int status);

/* Message describing the calling thread's most recent non-OK return. */
MOE_API const char* moe_last_error(void);

/*
 * moe_watchdog_trips - number of times, since the library was loaded on the
 * current device, that one of its kernels gave up on a barrier wait after the
 * wait's time limit (about 2 s) instead of spinning for ever.  A kernel that
 * trips the watchdog stops early and its outputs for that call are
 * unspecified.  Zero in normal operation.  Synchronises with the device (it is
 * a diagnostic, not for the hot path).  count: host pointer, out.
 */
MOE_API int moe_watchdog_trips(unsigned int* count);

/*
 * moe_topk_softmax - [R] §2: softmax over each row, top-k, optional
 * renormalise (the sgl_kernel topk_softmax(topk_weights, topk_ids,
 * gating_output, renormalize) call).
 *
 *   gating_output  device, (M, E) of `dtype` (MOE_DTYPE_F32 or MOE_DTYPE_BF16)
 *   M              rows, M >= 0
 *   E              experts, 1 <= E <= 1024
 *   topk           1 <= topk <= min(E, 32)
 *   renormalize    nonzero: weights divided by their sum
 *   topk_weights   device, (M, topk) fp32 out
 *   topk_ids       device, (M, topk) int32 out
 *   stream         cudaStream_t
 */
MOE_API int moe_topk_softmax(const void* gating_output, int dtype, int64_t M, int32_t E,
                     int32_t topk, int32_t renormalize, float* topk_weights,
                     int32_t* topk_ids, void* stream);

/*
 * moe_grouped_topk - [R] §3 (DeepSeek-V2 grouped_topk_gpu): softmax scores,
 * group score = the group's largest score, keep the topk_group best groups,
 * top-k over their experts, optional renormalise, then scale.
 *
 *   num_expert_group  G >= 1, G divides E
 *   topk_group        1 <= topk_group <= G
 *   topk              1 <= topk <= min(topk_group * E / G, 32)
 *   routed_scaling_factor  finite multiplier applied last (1.0 = none)
 *   other arguments as moe_topk_softmax
 */
MOE_API int moe_grouped_topk(const void* gating_output, int dtype, int64_t M, int32_t E,
                     int32_t topk, int32_t renormalize, int32_t num_expert_group,
                     int32_t topk_group, float routed_scaling_factor,
                     float* topk_weights, int32_t* topk_ids, void* stream);

/*
 * moe_grouped_topk_softcap - moe_grouped_topk with the logit softcapping of
 * the fused router ([R] §5: logits / c -> tanh -> * c when moe_softcapping is
 * nonzero).  c * tanh(x / c) is strictly increasing, so the experts chosen
 * are those of moe_grouped_topk; the weights are the softmax of the capped
 * logits (renormalised over the k or over all experts, then scaled).  With
 * topk = 1 and renormalize = 0 the weight is the top-1 probability
 * 1 / sum(exp(capped - capped max)) of the same section.  softcap 0 = none;
 * it must be finite.  Other arguments as moe_grouped_topk.
 */
MOE_API int moe_grouped_topk_softcap(const void* gating_output, int dtype, int64_t M, int32_t E, int32_t topk,
                                     int32_t renormalize, int32_t num_expert_group, int32_t topk_group,
                                     float routed_scaling_factor, float softcap, float* topk_weights,
                                     int32_t* topk_ids, void* stream);

/*
 * moe_biased_grouped_topk - [R] §4 (DeepSeek-V3 biased_grouped_topk_impl) and
 * [A] (aiter biased_grouped_topk): sigmoid scores; selection score = score +
 * correction_bias; group score = sum of the group's two largest selection
 * scores (a one-expert group: that score); keep the topk_group best groups;
 * top-k by selection score; weights are the unbiased sigmoid scores,
 * optionally renormalised, then scaled.  num_expert_group = topk_group = 1 is
 * the plain sigmoid(+bias) top-k of sgl_kernel topk_sigmoid.
 *
 *   correction_bias  device, (E,) fp32, or NULL for no bias.  It stays fp32
 *                    (the aiter path casts it to the logits dtype: see
 *                    moe_biased_grouped_topk_aiter).
 *   other arguments as moe_grouped_topk
 */
MOE_API int moe_biased_grouped_topk(const void* gating_output, int dtype,
                            const float* correction_bias, int64_t M, int32_t E,
                            int32_t topk, int32_t renormalize,
                            int32_t num_expert_group, int32_t topk_group,
                            float routed_scaling_factor, float* topk_weights,
                            int32_t* topk_ids, void* stream);

/*
 * moe_biased_grouped_topk_aiter - moe_biased_grouped_topk with the aiter
 * path's bias handling ([A] 코드 분석, After: aiter_biased_grouped_topk is
 * handed correction_bias.to(gating_output.dtype)): with bf16 logits the bias
 * is rounded to bf16 (round to nearest even) before it is added; with fp32
 * logits the two calls are identical.  Arguments as moe_biased_grouped_topk.
 */
MOE_API int moe_biased_grouped_topk_aiter(const void* gating_output, int dtype, const float* correction_bias,
                                          int64_t M, int32_t E, int32_t topk, int32_t renormalize,
                                          int32_t num_expert_group, int32_t topk_group,
                                          float routed_scaling_factor, float* topk_weights, int32_t* topk_ids,
                                          void* stream);

/*
 * moe_fused_router_workspace_size - bytes of device workspace that
 * moe_fused_router_topk needs for these sizes (0 when it needs none).  Small
 * batches (M <= 128) with a long hidden size (K >= 1024) spread K over up to
 * 256 CTAs whose fp32 partial logits meet in the workspace: (splits x M x
 * 256) floats, at most 2 MiB.  Returns (size_t)-1 for arguments
 * moe_fused_router_topk would reject.
 */
MOE_API size_t moe_fused_router_workspace_size(int64_t M, int32_t K, int32_t E);

/*
 * moe_fused_router_topk - [R] §5 (FusedMoeRouter) with the [R] §4 routing:
 * logits = hidden_states x router_weight accumulated in fp32 on the tensor
 * cores, then the moe_biased_grouped_topk routing of those logits.  From
 * M > 128 (or K < 1024) the logits stay on chip unless logits_out is given;
 * smaller batches with a long K pass fp32 partial logits through the
 * workspace to a second launch that sums and routes them.
 *
 *   hidden_states   device, (M, K) bf16
 *   router_weight   device, bf16, (K, E) if weight_layout == MOE_WEIGHT_K_BY_E
 *                   or (E, K) if MOE_WEIGHT_E_BY_K
 *   correction_bias device, (E,) fp32, or NULL
 *   M               tokens, below 2^31 (else MOE_ERR_UNSUPPORTED)
 *   K               hidden size, a positive multiple of 64
 *   E               experts; the fused router is built for E == 256
 *   logits_out      device, (M, E) fp32 out, or NULL (debug: the fp32 logits
 *                   the routing consumed)
 *   workspace       device scratch of at least
 *                   moe_fused_router_workspace_size(M, K, E) bytes, 256-byte
 *                   aligned (NULL allowed when that size is 0; otherwise a
 *                   missing or short workspace is MOE_ERR_INVALID_ARG).  No
 *                   initial contents are needed.  Calls that may overlap on
 *                   the GPU must not share one workspace.
 *   other arguments as moe_biased_grouped_topk
 */
MOE_API int moe_fused_router_topk(const void* hidden_states, const void* router_weight,
                          int weight_layout, const float* correction_bias,
                          int64_t M, int32_t K, int32_t E, int32_t topk,
                          int32_t renormalize, int32_t num_expert_group,
                          int32_t topk_group, float routed_scaling_factor,
                          float* topk_weights, int32_t* topk_ids,
                          float* logits_out, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * moe_fused_router_topk_noalloc - moe_fused_router_topk for callers that
 * cannot hand the library a workspace.  (The routing pages have no
 * counterpart to this call; it exists for the library's users.)
 *
 * Who needs it: code that is not allowed to allocate device memory at the
 * point where it routes tokens - inference engines that reserve every byte
 * of device memory during start-up and forbid allocations afterwards, or
 * plugin and embedding hosts that give the extension no allocator at all.
 * Batches of up to 128 tokens with a long hidden size need scratch memory
 * (moe_fused_router_workspace_size() > 0); this entry point takes it from a
 * fixed 2 MiB array compiled into the library instead of from the caller.
 *
 *   Arguments, layouts and results are those of moe_fused_router_topk,
 *   without `workspace` / `workspace_bytes`.
 *   Limit: none beyond moe_fused_router_topk's: the workspace of every size
 *   fits the array (moe_fused_router_workspace_size caps the partial logits
 *   at 2 MiB).  Batches above 128 tokens need no scratch.
 *   Memory: nothing is allocated or freed.  Every GPU that loads the library
 *   keeps the 2 MiB array for the life of the process.  The first call on
 *   each device looks up the array's device address (cudaGetSymbolAddress);
 *   make that first call before capturing the stream into a CUDA graph.
 *   Concurrency: all calls on a device share the one array, which keeps the
 *   last call's partial sums; calls that overlap on the GPU (different
 *   streams, or host threads racing on one device) race on it and give wrong
 *   results.  Serialise them (one stream), or use moe_fused_router_topk with a
 *   workspace per stream.
 */
MOE_API int moe_fused_router_topk_noalloc(const void* hidden_states, const void* router_weight,
                                          int weight_layout, const float* correction_bias, int64_t M,
                                          int32_t K, int32_t E, int32_t topk, int32_t renormalize,
                                          int32_t num_expert_group, int32_t topk_group,
                                          float routed_scaling_factor, float* topk_weights,
                                          int32_t* topk_ids, float* logits_out, void* stream);

/*
 * moe_fused_router_top1 - the fused top-1 router of [R] §5: per token row,
 *     l_e = sum_k h[k] * W(k, e)              (bf16 inputs, fp32 sums)
 *     id  = arg-max_e l_e                     (lower index among equal logits)
 *     w   = 1 / sum_e exp(cap(l_e) - cap(l_id)),  cap(x) = softcap * tanh(x / softcap)
 * i.e. softcapping (when softcap != 0; 0 = none), then top-1 with the
 * softmax probability of the chosen expert as its weight (the page's
 * invsumexp).  cap is increasing, so the arg-max of the raw logits is an
 * arg-max of the capped ones.
 *
 *   hidden_states   device, (M, K) bf16, 16-byte aligned
 *   router_weight   device, bf16, (K, E) if weight_layout == MOE_WEIGHT_K_BY_E
 *                   or (E, K) if MOE_WEIGHT_E_BY_K (the page's layout),
 *                   16-byte aligned
 *   K               hidden size, a positive multiple of 8 (of 64 for E > 8)
 *   E               experts, 1..256 (see the dispatch below)
 *   softcap         finite; 0 = no softcapping; c and -c give the same result
 *   topk_weights    device, (M, 1) fp32 out
 *   topk_ids        device, (M, 1) int32 out; -1 only if a kernel wait timed
 *                   out (moe_watchdog_trips counts it)
 *   logits_out      device, (M, E) fp32 out, or NULL (debug: the raw logits)
 * Dispatch: the tensor-core kernel (tcgen05, TMEM accumulator) when
 * K % 64 == 0, the layout is (E, K) and E <= 256, at every batch size (the
 * page switches to tensor cores from 512 tokens or E > 8; below that the
 * tensor-core kernel measured faster here too); otherwise the CUDA-core
 * kernel, which takes E <= 8 and K % 8 == 0.  E > 8 outside the tensor-core
 * conditions is MOE_ERR_UNSUPPORTED.
 * Asynchronous on `stream`; no allocation; M == 0 launches nothing.
 */
MOE_API int moe_fused_router_top1(const void* hidden_states, const void* router_weight, int weight_layout,
                                  int64_t M, int32_t K, int32_t E, float softcap, float* topk_weights,
                                  int32_t* topk_ids, float* logits_out, void* stream);

/*
 * moe_expert_permutation - the expert-sorted token permutation that follows
 * routing: the routing page's "Triton Kernels routing" branch hands the expert
 * runner RoutingData, GatherIndx and ScatterIndx (structure diagram 구조도 and
 * output format 출력 포맷: TRITON_KERNEL).  The page shows no body; this call
 * computes a stable counting sort of the M*k (token, slot) pairs of
 * topk_ids by expert id, with pair index i = token*k + slot.
 *
 *   topk_ids       int32 (M, k) row-major, device
 *   topk_weights   fp32 (M, k) or NULL (then gate_scal must be NULL too)
 *   expert_counts  int32 (E): pairs routed to each expert
 *   expert_offsets int32 (E + 1): exclusive prefix of the counts;
 *                  expert_offsets[E] = number of pairs with an id in [0, E)
 *   gather_indx    int32 (M*k): pair index at each sorted position (experts
 *                  ascending, pair index ascending within an expert); only
 *                  the first expert_offsets[E] entries are written
 *   scatter_indx   int32 (M*k): sorted position of each pair, -1 for a pair
 *                  whose id lies outside [0, E) (such pairs are skipped)
 *   gate_scal      fp32 (M*k) or NULL: topk_weights in sorted order
 *   workspace      device scratch of moe_expert_permutation_workspace_size()
 *                  bytes (no initial contents needed; owned by the caller, not
 *                  shared between calls that may run concurrently)
 * Deterministic: the same inputs give the same outputs bit for bit.
 * Limits: E <= 1024 and M*k < 2^31 (else MOE_ERR_UNSUPPORTED).  M = 0
 * writes zero counts and offsets.  Asynchronous on `stream`; no allocation.
 */
MOE_API size_t moe_expert_permutation_workspace_size(int64_t M, int32_t k, int32_t E);
MOE_API int moe_expert_permutation(const int32_t* topk_ids, const float* topk_weights, int64_t M, int32_t k,
                                   int32_t E, int32_t* expert_counts, int32_t* expert_offsets,
                                   int32_t* gather_indx, int32_t* scatter_indx, float* gate_scal,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_fill_shared_expert_slot - the shared-expert slot of the routing page
 * (§6 공유 전문가 슬롯 할당), applied in place to a finished routing result.
 *
 *   topk_weights, topk_ids  fp32 / int32 (M, k), device, row-major (in place)
 *   shared_pick    int32 (M,), device: the random draw per token, each value
 *                  in [0, num_shared) (the page uses torch.randint); values
 *                  outside that range are not checked
 *   routed_scaling_factor   0 = "None": the last slot's weight is left as it
 *                  is; otherwise it becomes (sum of the row's other k-1
 *                  weights, fp32 in slot order) / routed_scaling_factor
 * The last slot's id becomes E + shared_pick[row].  k <= 32; M = 0 is a no-op.
 */
MOE_API int moe_fill_shared_expert_slot(float* topk_weights, int32_t* topk_ids, int64_t M, int32_t k, int32_t E,
                                        int32_t num_shared, const int32_t* shared_pick,
                                        float routed_scaling_factor, void* stream);

/*
 * moe_fill_shared_expert_slot_philox - moe_fill_shared_expert_slot with the
 * random draw made by the library from a seed, so that a caller needs no
 * device-side random numbers of its own.  The routing page (§6) draws
 * torch.randint(E, E + num_shared) per token and names no generator; this
 * call uses Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC'11), a counter-based generator:
 *     u_i    = word 0 of Philox4x64-10(counter = (offset + i, carry, 0, 0),
 *                                      key = (seed, 0))
 *     pick_i = floor(u_i * num_shared / 2^64)         (in [0, num_shared))
 * for row i, the counter being offset + i as a 128-bit number.  The same
 * (seed, offset) always gives the same picks; advance offset by M between
 * calls for fresh draws.  Other arguments and the weight rule are those of
 * moe_fill_shared_expert_slot.  k <= 32; M = 0 is a no-op.
 */
MOE_API int moe_fill_shared_expert_slot_philox(float* topk_weights, int32_t* topk_ids, int64_t M, int32_t k,
                                               int32_t E, int32_t num_shared, uint64_t seed, uint64_t offset,
                                               float routed_scaling_factor, void* stream);

/*
 * moe_sort_topk_by_id - reorder every row's k (weight, id) pairs by ascending
 * id in place, equal ids keeping their order: the ascending id output that the
 * MiniMax-M3 page's minimax_decode_topk produces with a warp-wise rank sort
 * (코드 분석 §1).  k <= 32; M = 0 is a no-op.
 */
MOE_API int moe_sort_topk_by_id(float* topk_weights, int32_t* topk_ids, int64_t M, int32_t k, void* stream);

/*
 * moe_selftest_bounded_wait - checks the failure path of the library's
 * bounded waits without a fault: one thread waits on an mbarrier that nothing
 * completes, with a budget of budget_ns (0 < budget_ns <= 1e9), gives up and
 * writes status[0] = 1 (0 if the wait had completed) and status[1] = the
 * microseconds it waited.  status: device int32[2].  The routing kernels use
 * the same wait (with a 2 s budget) and count a give-up in
 * moe_watchdog_trips; this call touches no counter.
 */
MOE_API int moe_selftest_bounded_wait(uint64_t budget_ns, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTING_H */
