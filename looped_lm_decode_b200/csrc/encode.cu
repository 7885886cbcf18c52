// Encode: nearest-entry coding of loop-axis coupled vectors.
//
// LoopVQ paper, Sec. 4.1 eq. (4): the coupled vector of token n, channel group g
// takes channel g*c + i at loop step m of the block as coordinate i*Tc + m;
// Sec. 2 eq. (2): it is stored as the index of its nearest codebook entry.
// Sec. 4.3 "Encoding": a block is encoded once its last loop step exists.
//
// This direct kernel evaluates the squared distance to every entry in fp32,
// coordinate by coordinate in ascending order with separately rounded
// subtract / multiply / add, and keeps the first minimum, so its indices are the
// exact nearest entries under that arithmetic.  One thread owns one index word:
// the K and V codes of a channel group and of its RoPE partner group.
#include <math_constants.h>

#include "encode_common.cuh"

namespace loopvq {

struct EncodeArgs {
    const void *xk, *xv;
    int64_t s0, s1, s2, s3;   // element strides of (m, b, n, h)
    uint32_t *idx;            // words of (layer, block, b = 0, h = 0)
    const uint16_t *cb;       // codebook of (layer, block, kv = 0, h = 0): [2][Hkv][K][G]
    int Hkv, K, Nmax, b0, tok0, ntok;
};

template <typename XT>
__device__ __forceinline__ float ld_x(const XT *p);
template <>
__device__ __forceinline__ float ld_x<uint16_t>(const uint16_t *p) { return bf16_to_f32(__ldg(p)); }
template <>
__device__ __forceinline__ float ld_x<float>(const float *p) { return __ldg(p); }

template <int D, int C, int TC, typename XT>
__global__ void __launch_bounds__(128) encode_direct_kernel(const EncodeArgs a) {
    constexpr int G = C * TC;
    constexpr int NP = D / (2 * C);
    extern __shared__ __align__(16) float ecb[];           // [2][K][G] fp32: K codebook then V
    const int h = blockIdx.y;
    const int brel = blockIdx.z;
    const int b = a.b0 + brel;
    const int K = a.K;
    stage_codebooks<G>(ecb, a.cb, a.Hkv, h, K);
    __syncthreads();

    const int wl = blockIdx.x * blockDim.x + threadIdx.x;  // word within this (b, h) request
    if (wl >= a.ntok * NP) return;
    const int nrel = wl / NP;
    const int p = wl % NP;
    const int n = a.tok0 + nrel;

    // coupled vectors of groups p and p + NP, keys and values
    float z[4][G];
    const XT *xk = reinterpret_cast<const XT *>(a.xk);
    const XT *xv = reinterpret_cast<const XT *>(a.xv);
    const size_t base = (size_t)brel * a.s1 + (size_t)nrel * a.s2 + (size_t)h * a.s3;
#pragma unroll
    for (int m = 0; m < TC; ++m)
#pragma unroll
        for (int i = 0; i < C; ++i) {
            const size_t off = base + (size_t)m * a.s0;
            z[0][i * TC + m] = ld_x(xk + off + p * C + i);
            z[1][i * TC + m] = ld_x(xk + off + (p + NP) * C + i);
            z[2][i * TC + m] = ld_x(xv + off + p * C + i);
            z[3][i * TC + m] = ld_x(xv + off + (p + NP) * C + i);
        }
    const uint32_t word = nearest_word<G>(z, ecb, ecb + (size_t)K * G, K);
    a.idx[((size_t)b * a.Hkv + h) * idx_words_per_bh(a.Nmax, D, C) + idx_word(n, p, NP)] = word;
}

// One codebook per channel group: a CTA takes one pair-group p of one head and stages the four
// codebooks its words use (K and V of groups p and p + NP); one thread per token writes its word.
// Grid: (ceil(ntok / 128), NP * Hkv, nb).
template <int D, int C, int TC, typename XT>
__global__ void __launch_bounds__(128) encode_pg_kernel(const EncodeArgs a) {
    constexpr int G = C * TC;
    constexpr int NP = D / (2 * C);
    constexpr int NCB = D / C;
    extern __shared__ __align__(16) float ecb[];           // [4][K][G]: K_p, K_{p+NP}, V_p, V_{p+NP}
    const int p = blockIdx.y % NP, h = blockIdx.y / NP;
    const int brel = blockIdx.z;
    const int b = a.b0 + brel;
    const int K = a.K;
    for (int e = threadIdx.x; e < 4 * K * G; e += blockDim.x) {
        const int which = e / (K * G);
        const int rem = e % (K * G);
        const int kv = which >> 1, g = (which & 1) ? p + NP : p;
        ecb[e] = bf16_to_f32(a.cb[(((size_t)kv * a.Hkv + h) * NCB + g) * (size_t)K * G + rem]);
    }
    __syncthreads();
    const int nrel = blockIdx.x * blockDim.x + threadIdx.x;
    if (nrel >= a.ntok) return;
    float z[4][G];
    const XT *xk = reinterpret_cast<const XT *>(a.xk);
    const XT *xv = reinterpret_cast<const XT *>(a.xv);
    const size_t base = (size_t)brel * a.s1 + (size_t)nrel * a.s2 + (size_t)h * a.s3;
#pragma unroll
    for (int m = 0; m < TC; ++m)
#pragma unroll
        for (int i = 0; i < C; ++i) {
            const size_t off = base + (size_t)m * a.s0;
            z[0][i * TC + m] = ld_x(xk + off + p * C + i);
            z[1][i * TC + m] = ld_x(xk + off + (p + NP) * C + i);
            z[2][i * TC + m] = ld_x(xv + off + p * C + i);
            z[3][i * TC + m] = ld_x(xv + off + (p + NP) * C + i);
        }
    const size_t KG = (size_t)K * G;
    const uint32_t word = nearest_word4<G>(z, ecb, ecb + KG, ecb + 2 * KG, ecb + 3 * KG, K);
    a.idx[((size_t)b * a.Hkv + h) * idx_words_per_bh(a.Nmax, D, C) + idx_word(a.tok0 + nrel, p, NP)] = word;
}

template <int D, int C, int TC>
static cudaError_t launch_ct(const EncodeArgs &a, int x_dtype, int nb, bool pg, cudaStream_t s) {
    constexpr int NP = D / (2 * C);
    if (pg) {
        const size_t smem = 4 * (size_t)a.K * C * TC * sizeof(float);
        dim3 grid((a.ntok + 127) / 128, NP * a.Hkv, nb);
        auto k = x_dtype == LOOPVQ_BF16 ? encode_pg_kernel<D, C, TC, uint16_t> : encode_pg_kernel<D, C, TC, float>;
        cudaError_t e = ensure_dynamic_smem((const void *)k, smem);
        if (e != cudaSuccess) return e;
        k<<<grid, 128, smem, s>>>(a);
        return cudaGetLastError();
    }
    const size_t smem = 2 * (size_t)a.K * C * TC * sizeof(float);
    dim3 grid((a.ntok * NP + 127) / 128, a.Hkv, nb);
    if (x_dtype == LOOPVQ_BF16) {
        auto k = encode_direct_kernel<D, C, TC, uint16_t>;
        cudaError_t e = ensure_dynamic_smem((const void *)k, smem);
        if (e != cudaSuccess) return e;
        k<<<grid, 128, smem, s>>>(a);
    } else {
        auto k = encode_direct_kernel<D, C, TC, float>;
        cudaError_t e = ensure_dynamic_smem((const void *)k, smem);
        if (e != cudaSuccess) return e;
        k<<<grid, 128, smem, s>>>(a);
    }
    return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_c(int c, int tc, const EncodeArgs &a, int x_dtype, int nb, bool pg, cudaStream_t s) {
    if (c == 4) {
        if (tc == 4) return launch_ct<D, 4, 4>(a, x_dtype, nb, pg, s);
        if (tc == 2) return launch_ct<D, 4, 2>(a, x_dtype, nb, pg, s);
        if (tc == 1) return launch_ct<D, 4, 1>(a, x_dtype, nb, pg, s);
    } else if (c == 8) {
        if (tc == 4) return launch_ct<D, 8, 4>(a, x_dtype, nb, pg, s);
        if (tc == 2) return launch_ct<D, 8, 2>(a, x_dtype, nb, pg, s);
        if (tc == 1) return launch_ct<D, 8, 1>(a, x_dtype, nb, pg, s);
    } else if (c == 16) {
        if (tc == 2) return launch_ct<D, 16, 2>(a, x_dtype, nb, pg, s);
        if (tc == 1) return launch_ct<D, 16, 1>(a, x_dtype, nb, pg, s);
    } else if (c == 32) {
        if (tc == 1) return launch_ct<D, 32, 1>(a, x_dtype, nb, pg, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_encode_tc(const loopvq_cache &cc, int layer, int block, const void *xk, const void *xv,
                             const int64_t *strides, int b0, int nb, int tok0, int ntok, cudaStream_t s);

cudaError_t launch_encode(const loopvq_cache &cc, int layer, int block, const void *xk, const void *xv,
                          int x_dtype, const int64_t *strides, int b0, int nb, int tok0, int ntok,
                          cudaStream_t s) {
    if (nb == 0 || ntok == 0) return cudaSuccess;
    // bf16 inputs with a tensor-core instantiation (shared or per-group codebooks) go to the tcgen05
    // contraction; fp32 inputs (not representable as bf16 MMA operands) and other shapes use the exact
    // CUDA-core kernels below
    if (x_dtype == LOOPVQ_BF16) {
        const cudaError_t e = launch_encode_tc(cc, layer, block, xk, xv, strides, b0, nb, tok0, ntok, s);
        if (e != cudaErrorNotSupported) return e;
    }
    EncodeArgs a{};
    a.xk = xk;
    a.xv = xv;
    a.s0 = strides[0];
    a.s1 = strides[1];
    a.s2 = strides[2];
    a.s3 = strides[3];
    a.idx = cc.idx + idx_base(cc, layer, block, 0, 0);
    a.cb = cc.codebook + codebook_base(cc, layer, block, 0, 0);
    a.Hkv = cc.Hkv;
    a.K = cc.K;
    a.Nmax = cc.Nmax;
    a.b0 = b0;
    a.tok0 = tok0;
    a.ntok = ntok;
    const bool pg = ncb_of(cc) > 1;
    if (cc.D == 128) return dispatch_c<128>(cc.c, cc.Tc, a, x_dtype, nb, pg, s);
    if (cc.D == 64) return dispatch_c<64>(cc.c, cc.Tc, a, x_dtype, nb, pg, s);
    return cudaErrorInvalidValue;
}

}  // namespace loopvq
