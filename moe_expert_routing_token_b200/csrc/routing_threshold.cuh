// Threshold network shared by the direct and the two-phase routing kernels:
// the K-th largest of the values that a row's eight lanes hold two each.
#pragma once

#include "routing_common.cuh"

namespace moe {

// The K-th largest (1 <= K <= 8) and the largest of the 16 values held two
// per lane, t0 >= t1, by the eight lanes of a row: the xor-1
// exchange makes sorted 4-lists ([t0, t1, p1, p0] is bitonic), the xor-2
// exchange sorted 8-lists, and the xor-4 exchange the top 8 of the 16 (the
// elementwise maximum against the reversed partner, a bitonic sequence that
// is sorted only when K < 8 needs it).
template <int L>
__device__ __forceinline__ float row_kth2(float t0, float t1, int K, float& vmax) {
    static_assert(L == 8, "two values per lane on eight lanes");
    float a[8];
    {
        float x[4] = {t0, t1, __shfl_xor_sync(kFullMask, t1, 1), __shfl_xor_sync(kFullMask, t0, 1)};
        bitonic_clean_desc(x);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[i] = x[i];
            a[7 - i] = __shfl_xor_sync(kFullMask, x[i], 2);
        }
        bitonic_clean_desc(a);
        float b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = __shfl_xor_sync(kFullMask, a[i], 4);
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fmaxf(a[i], b[7 - i]);
    }
    vmax = fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
    if (K == 8) return fminf(fminf(fminf(a[0], a[1]), fminf(a[2], a[3])), fminf(fminf(a[4], a[5]), fminf(a[6], a[7])));
    bitonic_clean_desc(a);
    return kth_of_sorted8(a, K);
}

}  // namespace moe
