// Exact nearest-entry coding shared by the prefill encoder (encode.cu) and the decode-time page
// encoder (window.cu).
//
// LoopVQ paper, Sec. 2 eq. (2): a coupled vector is stored as the index of its nearest codebook
// entry under the squared Euclidean distance; the lowest index wins ties.
#pragma once

#include <math_constants.h>

#include "loopvq_internal.cuh"

namespace loopvq {

// Exact fp32 nearest entries of the four coupled vectors of one index word (keys of groups p and
// p + NP, values of the same groups): distances accumulated over the coordinates in ascending order
// with separately rounded subtract, multiply and add; the first minimum is kept.  ek, ev: the K and
// V codebooks of the head as fp32 [K][G].
// Exact fp32 nearest entries of the four coupled vectors of one index word, each in its own codebook
// (fp32 [K][G]): distances accumulated over the coordinates in ascending order with separately
// rounded subtract, multiply and add; the first minimum is kept.
template <int G>
__device__ __forceinline__ uint32_t nearest_word4(const float (&z)[4][G], const float *e0, const float *e1,
                                                  const float *e2, const float *e3, int K) {
    float best[4] = {CUDART_INF_F, CUDART_INF_F, CUDART_INF_F, CUDART_INF_F};
    int bi[4] = {0, 0, 0, 0};
    for (int r = 0; r < K; ++r) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < G; ++k) {
            float t;
            t = __fsub_rn(z[0][k], e0[r * G + k]); d[0] = __fadd_rn(d[0], __fmul_rn(t, t));
            t = __fsub_rn(z[1][k], e1[r * G + k]); d[1] = __fadd_rn(d[1], __fmul_rn(t, t));
            t = __fsub_rn(z[2][k], e2[r * G + k]); d[2] = __fadd_rn(d[2], __fmul_rn(t, t));
            t = __fsub_rn(z[3][k], e3[r * G + k]); d[3] = __fadd_rn(d[3], __fmul_rn(t, t));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (d[u] < best[u]) { best[u] = d[u]; bi[u] = r; }
    }
    return (uint32_t)bi[0] | ((uint32_t)bi[1] << 8) | ((uint32_t)bi[2] << 16) | ((uint32_t)bi[3] << 24);
}

// The same with one codebook for the keys (groups p and p + NP) and one for the values.
template <int G>
__device__ __forceinline__ uint32_t nearest_word(const float (&z)[4][G], const float *ek, const float *ev, int K) {
    return nearest_word4<G>(z, ek, ek, ev, ev, K);
}

// Stage the head's K and V codebooks as fp32 [2][K][G] in shared memory.
template <int G>
__device__ __forceinline__ void stage_codebooks(float *ecb, const uint16_t *cb, int Hkv, int h, int K) {
    for (int e = threadIdx.x; e < 2 * K * G; e += blockDim.x) {
        const int kv = e / (K * G);
        const int rem = e % (K * G);
        ecb[e] = bf16_to_f32(cb[((size_t)kv * Hkv + h) * (size_t)K * G + rem]);
    }
}

}  // namespace loopvq
