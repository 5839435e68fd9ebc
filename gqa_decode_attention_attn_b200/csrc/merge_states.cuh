// merge_states.cuh -- standalone exact merge of S partial softmax states per row
// (LeanAttention decode tiles digest, section "Exact softmax that merges piece
// by piece": each piece keeps its own maximum, normaliser and weighted values;
// rescaling them to the common maximum and adding is exact in any order).
//
// One warp per row.  Lanes stride the D columns; the pieces are visited in
// index order so the result does not depend on scheduling.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace gqa {

constexpr int MERGE_WARPS = 8;

__global__ void __launch_bounds__(MERGE_WARPS * 32)
    merge_states_kernel(const float *__restrict__ acc, const float *__restrict__ m,
                        const float *__restrict__ l, int S, int N, int D,
                        uint16_t *__restrict__ out, float *__restrict__ lse)
{
    const int lane = threadIdx.x & 31;
    const int64_t n = (int64_t)blockIdx.x * MERGE_WARPS + (threadIdx.x >> 5);
    if (n >= N)
        return;
    float ms = -INFINITY;
    for (int i = lane; i < S; i += 32)
        ms = fmaxf(ms, m[(int64_t)i * N + n]);
#pragma unroll
    for (int o = 16; o; o >>= 1)
        ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
    // Normaliser: every lane sums all pieces in the same order (no reduction
    // tree), so each lane holds the identical value.
    float ls = 0.f;
    for (int i = 0; i < S; ++i) {
        const float mi = m[(int64_t)i * N + n];
        const float w = mi == -INFINITY ? 0.f : expf(mi - ms);
        ls = fmaf(w, l[(int64_t)i * N + n], ls);
    }
    for (int d = lane; d < D; d += 32) {
        float a = 0.f;
        for (int i = 0; i < S; ++i) {
            const float mi = m[(int64_t)i * N + n];
            const float w = mi == -INFINITY ? 0.f : expf(mi - ms);
            a = fmaf(w, acc[((int64_t)i * N + n) * D + d], a);
        }
        const float o = ls > 0.f ? a / ls : 0.f;
        __nv_bfloat16 h = __float2bfloat16_rn(o);
        out[n * D + d] = *reinterpret_cast<uint16_t *>(&h);
    }
    if (lse && lane == 0)
        lse[n] = ls > 0.f ? ms + logf(ls) : -INFINITY;
}

}  // namespace gqa
