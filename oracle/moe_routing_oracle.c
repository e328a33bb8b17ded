/*
 * Plain CPU oracle for Mixture-of-Experts token-to-expert routing.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * Style: one row at a time, one step at a time, in double precision, in the
 * order the pages give the steps.  The only library primitives used are
 * exp(), tanh() and qsort().  There is deliberately no blocking, fusion or
 * cleverness.
 *
 * Sources (pages on SGLang MoE routing; cited by page title and section):
 *   [M] "MiniMax-M3 모델을 위한 FP8 Attention GEMM 최적화 및 성능 개선"
 *       코드 분석 §1 minimax_decode_topk - ascending (sorted) id output
 *   [R] "[SGLang] MoE 라우팅: 토큰에서 전문가로의 배분 알고리즘"
 *       (SGLang MoE routing: token-to-expert algorithms)
 *       §2 기본 softmax Top-K     - softmax scores, top-k, renormalise
 *       §3 Grouped Top-K          - group score = max of the group's scores,
 *                                   keep the topk_group best groups, mask the
 *                                   rest, top-k over the survivors
 *       §4 Biased Grouped Top-K   - sigmoid scores, correction_bias added for
 *                                   the choice, group score = sum of the top-2
 *                                   biased scores in the group
 *       §5 Fused MoE Router       - logits = hidden_states x router weight in
 *                                   fp32 accumulation, optional softcapping
 *                                   c * tanh(logits / c), routing on the result
 *       §6 공유 전문가 슬롯 할당       - the last slot goes to a shared expert
 *   [A] "[sglang] SGLang MoE 라우팅 최적화: AMD GPU에서 aiter.biased_grouped_topk 활용"
 *       코드 분석 (After)           - sigmoid + correction_bias routing expressed
 *                                   as biased grouped top-k with
 *                                   num_expert_group = 1, topk_group = 1
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - ties between experts or between groups: the lower index wins;
 *   - ids are emitted in descending selection score (lower index first on ties);
 *   - experts of unselected groups are excluded (equivalent to a -inf mask);
 *   - renormalise divides the k gathered weights by their sum, then the
 *     routed scaling factor multiplies them;
 *   - the gathered weight is the unbiased score (the bias only steers choice);
 *   - a group of one expert has that expert's score as its top-2 sum.
 *
 * Parity pins: see tests/test_oracle_*.py (hand-worked closed forms, brute
 * force over all subsets, library cross-checks, invariants, and source
 * mutants that the pins must reject).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#define ORACLE_SOFTMAX 0
#define ORACLE_SIGMOID 1
#define ORACLE_GROUP_MAX 0
#define ORACLE_GROUP_TOP2_SUM 1

#define ORACLE_OK 0
#define ORACLE_BAD_ARGS 1
#define ORACLE_NO_MEMORY 2

/* ---------------------------------------------------------------------------
 * Sorting helper: an (value, index) pair ordered by value descending, then by
 * index ascending.  This is the whole tie-break rule.
 * ------------------------------------------------------------------------- */
typedef struct {
    double value;
    int index;
} ranked_t;

static int by_value_desc_then_index_asc(const void* pa, const void* pb) {
    const ranked_t* a = (const ranked_t*)pa;
    const ranked_t* b = (const ranked_t*)pb;
    if (a->value > b->value) return -1;
    if (a->value < b->value) return 1;
    if (a->index < b->index) return -1;
    if (a->index > b->index) return 1;
    return 0;
}

/* ---------------------------------------------------------------------------
 * Step 1 - scores.  [R] §2 (softmax over the row) and [R] §4 (sigmoid).
 * ------------------------------------------------------------------------- */
static void score_row(const double* x, int E, int scoring, double* p) {
    if (scoring == ORACLE_SOFTMAX) {
        double mx = x[0];
        for (int e = 1; e < E; ++e)
            if (x[e] > mx) mx = x[e];
        double sum = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp(x[e] - mx);
            sum += p[e];
        }
        for (int e = 0; e < E; ++e) p[e] = p[e] / sum;
    } else {
        for (int e = 0; e < E; ++e) p[e] = 1.0 / (1.0 + exp(-x[e]));
    }
}

/* ---------------------------------------------------------------------------
 * Step 3 - group score of experts [g*S, (g+1)*S).
 *   max       : [R] §3, the largest score in the group;
 *   top-2 sum : [R] §4, the sum of the two largest biased scores in the group.
 * ------------------------------------------------------------------------- */
static double group_score(const double* s, int first, int S, int kind) {
    if (kind == ORACLE_GROUP_MAX) {
        double m = s[first];
        for (int j = 1; j < S; ++j)
            if (s[first + j] > m) m = s[first + j];
        return m;
    }
    /* sum of the two largest values (a group of one: that value alone) */
    double best = s[first];
    int best_j = 0;
    for (int j = 1; j < S; ++j)
        if (s[first + j] > best) {
            best = s[first + j];
            best_j = j;
        }
    if (S == 1) return best;
    double second = -INFINITY;
    for (int j = 0; j < S; ++j)
        if (j != best_j && s[first + j] > second) second = s[first + j];
    return best + second;
}

/* ---------------------------------------------------------------------------
 * oracle_route: route M rows of logits (row-major, M x E, given as doubles
 * holding the exact stored input values).
 *
 *   scoring      ORACLE_SOFTMAX or ORACLE_SIGMOID
 *   bias         E values added to the scores for the choice only, or NULL
 *   G, TG        num_expert_group and topk_group (G divides E; 1 <= TG <= G)
 *   group_kind   ORACLE_GROUP_MAX or ORACLE_GROUP_TOP2_SUM
 *   k            experts per token (1 <= k <= TG * E / G)
 *   renorm       nonzero: divide the gathered weights by their sum
 *   rsf          routed scaling factor, multiplied in last
 * Outputs (row-major):
 *   ids      M x k   expert ids, descending selection score
 *   weights  M x k   the gathered unbiased scores after renorm and scaling
 *   scores   M x E   unbiased scores p (NULL to skip)
 *   sel      M x E   selection scores s = p + bias (NULL to skip)
 *   gsc      M x G   group scores (NULL to skip)
 *   margins  M x 3   [0] s_(k) - s_(k+1) over the admissible experts
 *                        (+inf when fewer than k+1 are admissible)
 *                    [1] gs_(TG) - gs_(TG+1) over the groups (+inf if TG == G)
 *                    [2] smallest gap between consecutive selected scores
 *                        (+inf when k == 1)
 *                    (NULL to skip)
 * Returns ORACLE_OK, ORACLE_BAD_ARGS or ORACLE_NO_MEMORY.
 * ------------------------------------------------------------------------- */
int oracle_route(const double* logits, int64_t M, int E, int scoring,
                 const double* bias, int G, int TG, int group_kind, int k,
                 int renorm, double rsf, int32_t* ids, double* weights,
                 double* scores, double* sel, double* gsc, double* margins) {
    if (M < 0 || E < 1 || G < 1 || E % G != 0 || TG < 1 || TG > G || k < 1)
        return ORACLE_BAD_ARGS;
    const int S = E / G;
    if (k > TG * S) return ORACLE_BAD_ARGS;
    if (scoring != ORACLE_SOFTMAX && scoring != ORACLE_SIGMOID) return ORACLE_BAD_ARGS;
    if (group_kind != ORACLE_GROUP_MAX && group_kind != ORACLE_GROUP_TOP2_SUM)
        return ORACLE_BAD_ARGS;

    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    ranked_t* groups = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)G);
    ranked_t* admissible = (ranked_t*)malloc(sizeof(ranked_t) * (size_t)E);
    int* group_kept = (int*)malloc(sizeof(int) * (size_t)G);
    if (!p || !s || !groups || !admissible || !group_kept) {
        free(p); free(s); free(groups); free(admissible); free(group_kept);
        return ORACLE_NO_MEMORY;
    }

    for (int64_t i = 0; i < M; ++i) {
        const double* x = logits + i * (int64_t)E;

        /* 1. scores */
        score_row(x, E, scoring, p);
        if (scores)
            for (int e = 0; e < E; ++e) scores[i * (int64_t)E + e] = p[e];

        /* 2. selection scores: bias steers the choice only ([R] §4) */
        for (int e = 0; e < E; ++e) s[e] = p[e] + (bias ? bias[e] : 0.0);
        if (sel)
            for (int e = 0; e < E; ++e) sel[i * (int64_t)E + e] = s[e];

        /* 3. group scores */
        for (int g = 0; g < G; ++g) {
            groups[g].value = group_score(s, g * S, S, group_kind);
            groups[g].index = g;
            if (gsc) gsc[i * (int64_t)G + g] = groups[g].value;
        }

        /* 4. keep the TG best groups ([R] §3) */
        qsort(groups, (size_t)G, sizeof(ranked_t), by_value_desc_then_index_asc);
        for (int g = 0; g < G; ++g) group_kept[g] = 0;
        for (int t = 0; t < TG; ++t) group_kept[groups[t].index] = 1;

        /* 5. top-k over the experts of the kept groups */
        int n_adm = 0;
        for (int e = 0; e < E; ++e) {
            if (group_kept[e / S]) {
                admissible[n_adm].value = s[e];
                admissible[n_adm].index = e;
                ++n_adm;
            }
        }
        qsort(admissible, (size_t)n_adm, sizeof(ranked_t), by_value_desc_then_index_asc);

        /* 6. gather the unbiased scores, renormalise, scale */
        double wsum = 0.0;
        for (int j = 0; j < k; ++j) {
            ids[i * (int64_t)k + j] = (int32_t)admissible[j].index;
            weights[i * (int64_t)k + j] = p[admissible[j].index];
            wsum += p[admissible[j].index];
        }
        for (int j = 0; j < k; ++j) {
            double w = weights[i * (int64_t)k + j];
            if (renorm) w = w / wsum;
            weights[i * (int64_t)k + j] = w * rsf;
        }

        if (margins) {
            double* mg = margins + i * 3;
            mg[0] = (n_adm > k) ? admissible[k - 1].value - admissible[k].value : INFINITY;
            mg[1] = (G > TG) ? groups[TG - 1].value - groups[TG].value : INFINITY;
            double gap = INFINITY;
            for (int j = 0; j + 1 < k; ++j) {
                double d = admissible[j].value - admissible[j + 1].value;
                if (d < gap) gap = d;
            }
            mg[2] = gap;
        }
    }

    free(p); free(s); free(groups); free(admissible); free(group_kept);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * oracle_router_logits: the router projection of [R] §5 for M rows.
 *   logits[i][e] = sum over c of h[i][c] * W(c, e), summed in double in
 *   ascending c.  Inputs are the exact stored bf16 values as doubles, so every
 *   product is exact and only the summation rounds.
 *   w_layout 0: W stored (K, E) row-major, W(c, e) = w[c*E + e]
 *   w_layout 1: W stored (E, K) row-major, W(c, e) = w[e*K + c]
 * ------------------------------------------------------------------------- */
int oracle_router_logits(const double* h, const double* w, int64_t M, int K, int E,
                         int w_layout, double* logits) {
    if (M < 0 || K < 1 || E < 1 || (w_layout != 0 && w_layout != 1)) return ORACLE_BAD_ARGS;
    for (int64_t i = 0; i < M; ++i) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int c = 0; c < K; ++c) {
                double wv = (w_layout == 0) ? w[(int64_t)c * E + e] : w[(int64_t)e * K + c];
                acc += h[i * (int64_t)K + c] * wv;
            }
            logits[i * (int64_t)E + e] = acc;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * oracle_softcap: the logit softcapping of [R] §5 (the fused router's
 * Softcapping step), out[i] = c * tanh(x[i] / c) for n values.  The page
 * applies it only when the softcapping constant is nonzero; c == 0 copies the
 * values unchanged.  c and -c give the same values (tanh is odd); c must be
 * finite.  x and out may be the same array.
 * ------------------------------------------------------------------------- */
int oracle_softcap(const double* x, int64_t n, double c, double* out) {
    if (n < 0 || c != c || c == INFINITY || c == -INFINITY) return ORACLE_BAD_ARGS;
    for (int64_t i = 0; i < n; ++i) {
        if (c == 0.0)
            out[i] = x[i];
        else
            out[i] = c * tanh(x[i] / c);
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * oracle_expert_permutation: the expert-sorted token permutation that the
 * routing page's "Triton Kernels routing" branch hands to the expert runner
 * ([R] 구조도, 출력 포맷: RoutingData, GatherIndx, ScatterIndx).  The pages give
 * only the names; the reading taken is a stable counting sort of the M*k
 * (token, slot) pairs by expert id, pair index i = token*k + slot:
 *   counts[e]      number of pairs routed to expert e
 *   offsets[e]     sum of counts[0..e), offsets[E] = M*k
 *   gather[p]      the pair index at sorted position p (experts ascending,
 *                  pair index ascending within an expert)
 *   scatter[i]     the sorted position of pair i (gather[scatter[i]] == i)
 *   gate[p]        weights[gather[p]] (NULL weights or gate: skipped)
 * A pair whose id lies outside [0, E) is skipped: not counted, not placed,
 * scatter = -1 (offsets[E] is then the number of placed pairs).  Reason: the
 * routing page's shared-expert slot (§6, 공유 전문가 슬롯 할당) writes ids
 * E .. E + n_shared - 1 into topk_ids, so a routing result handed to a
 * permutation over the E routed experts can carry ids that name no expert of
 * that sort; those pairs get no position.  A negative id (a pair masked out
 * before this step) is read the same way.
 * ------------------------------------------------------------------------- */
int oracle_expert_permutation(const int32_t* ids, const double* weights, int64_t M, int k, int E,
                              int32_t* counts, int32_t* offsets, int32_t* gather, int32_t* scatter,
                              double* gate) {
    if (M < 0 || k < 1 || E < 1) return ORACLE_BAD_ARGS;
    const int64_t n = M * (int64_t)k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n; ++i)
        if (ids[i] >= 0 && ids[i] < E) counts[ids[i]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    if (!cursor) return ORACLE_NO_MEMORY;
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t i = 0; i < n; ++i) {       /* pairs in ascending index: stable */
        if (ids[i] < 0 || ids[i] >= E) {
            scatter[i] = -1;
            continue;
        }
        const int32_t p = cursor[ids[i]]++;
        gather[p] = (int32_t)i;
        scatter[i] = p;
        if (weights && gate) gate[p] = weights[i];
    }
    free(cursor);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * oracle_fill_shared_slot: the shared-expert slot of [R] §6 (공유 전문가 슬롯
 * 할당) on a finished routing result (weights, ids: M x k, in place).  The
 * last slot of every row gets the shared expert E + pick[i] (pick[i] in
 * [0, num_shared): the random draw, passed in); when rsf != 0 its weight
 * becomes the sum of the row's other k-1 weights divided by rsf (rsf == 0:
 * "routed_scaling_factor is None", the weight is left as it is).
 * ------------------------------------------------------------------------- */
int oracle_fill_shared_slot(double* weights, int32_t* ids, int64_t M, int k, int E, int num_shared,
                            const int32_t* pick, double rsf) {
    if (M < 0 || k < 1 || E < 1 || num_shared < 1) return ORACLE_BAD_ARGS;
    for (int64_t i = 0; i < M; ++i) {
        if (pick[i] < 0 || pick[i] >= num_shared) return ORACLE_BAD_ARGS;
        ids[i * (int64_t)k + (k - 1)] = E + pick[i];
        if (rsf != 0.0) {
            double sum = 0.0;
            for (int j = 0; j < k - 1; ++j) sum += weights[i * (int64_t)k + j];
            weights[i * (int64_t)k + (k - 1)] = sum / rsf;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * oracle_philox4x64: the Philox4x64-10 counter-based generator of Salmon,
 * Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3"
 * (SC'11).  Ten rounds on a counter of four 64-bit words under a key of two;
 * a round multiplies words 0 and 2 by the two Philox constants and forms
 *   (hi(M1 x2) ^ x1 ^ k0,  lo(M1 x2),  hi(M0 x0) ^ x3 ^ k1,  lo(M0 x0)),
 * and the key is bumped by the two Weyl constants before every round but the
 * first.  out may not alias ctr.
 * ------------------------------------------------------------------------- */
void oracle_philox4x64(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
    uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += W0;
            k1 += W1;
        }
        const unsigned __int128 p0 = (unsigned __int128)M0 * x0;
        const unsigned __int128 p1 = (unsigned __int128)M1 * x2;
        const uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
        const uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
        const uint64_t y0 = hi1 ^ x1 ^ k0, y1 = lo1, y2 = hi0 ^ x3 ^ k1, y3 = lo0;
        x0 = y0;
        x1 = y1;
        x2 = y2;
        x3 = y3;
    }
    out[0] = x0;
    out[1] = x1;
    out[2] = x2;
    out[3] = x3;
}

/* ---------------------------------------------------------------------------
 * oracle_shared_pick_philox: the random shared-expert draw of [R] §6
 * (torch.randint(num_experts, num_experts + num_fused_shared_experts), one
 * per token) made reproducible from a seed.  The pages name no generator;
 * the reading taken: token i draws u = word 0 of Philox4x64-10 with counter
 * (offset + i as a 128-bit number in words 0-1, 0, 0) and key (seed, 0), and
 * picks floor(u * num_shared / 2^64), the high word of the 128-bit product.
 * ------------------------------------------------------------------------- */
int oracle_shared_pick_philox(int64_t M, int num_shared, uint64_t seed, uint64_t offset, int32_t* pick) {
    if (M < 0 || num_shared < 1) return ORACLE_BAD_ARGS;
    const uint64_t key[2] = {seed, 0};
    for (int64_t i = 0; i < M; ++i) {
        const uint64_t c0 = offset + (uint64_t)i;
        const uint64_t ctr[4] = {c0, c0 < offset ? 1u : 0u, 0, 0};
        uint64_t out[4];
        oracle_philox4x64(ctr, key, out);
        pick[i] = (int32_t)(uint64_t)(((unsigned __int128)out[0] * (uint64_t)num_shared) >> 64);
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * oracle_sort_by_id: reorder every row's k (weight, id) pairs by ascending
 * id, equal ids keeping their order - the ascending expert/block-id output
 * that [M] 코드 분석 §1 (minimax_decode_topk) produces with a warp rank sort.
 * ------------------------------------------------------------------------- */
int oracle_sort_by_id(double* weights, int32_t* ids, int64_t M, int k) {
    if (M < 0 || k < 1) return ORACLE_BAD_ARGS;
    for (int64_t i = 0; i < M; ++i) {
        int32_t* id = ids + i * (int64_t)k;
        double* w = weights + i * (int64_t)k;
        for (int a = 1; a < k; ++a) {          /* insertion sort: stable */
            const int32_t ka = id[a];
            const double wa = w[a];
            int b = a - 1;
            while (b >= 0 && id[b] > ka) {
                id[b + 1] = id[b];
                w[b + 1] = w[b];
                --b;
            }
            id[b + 1] = ka;
            w[b + 1] = wa;
        }
    }
    return ORACLE_OK;
}
