// TaSQ before loop-axis coupling: the token scales and the encoder.
//
// LoopVQ paper, App. B "Formulation": the pre-RoPE key of loop step t is mapped to
// u = P(w (.) k / sigma), with w a per-channel weight, sigma the root mean square of w (.) k over
// all heads and channels of the token, and P a channel permutation; the coupled key vectors (4)
// are built from u.  "Grouping under loop coupling": a code holds complete RoPE pairs
// {f, f + D/2} at all Tc loop steps of the block.  "Calibration and bitwidth": sigma is kept in
// fp16.
//
// sigma: one warp per (token, loop step, sequence); the squares of w * k are summed in fp64
// without fused multiply-adds, reduced across the warp, and the root mean square is rounded to
// fp16.  The encoder is the exact fp32 nearest-entry coder of encode_common.cuh on the coupled
// vectors of u (w * k rounded, divided by the fp16 sigma, rounded) for the keys, and of the plain
// values: the index word (token, p) holds the key codes of TaSQ groups 2p and 2p + 1 and the value
// codes of channel groups p and p + NP.
#include <cuda_fp16.h>

#include "encode_common.cuh"

namespace loopvq {

struct TasqArgs {
    const void *xk, *xv;
    int64_t s0, s1, s2, s3;      // element strides of (m, b - b0, n - tok0, h)
    const float *w;              // weights of (layer, t = block * Tc): [Tc][Hkv][D]
    const int16_t *perm;         // order of (layer, block): [Hkv][D/2]
    uint16_t *sigma;             // scales of (layer, t = block * Tc): [Tc][B][Nmax]
    uint32_t *idx;               // words of (layer, block, b = 0, h = 0)
    const uint16_t *cb;          // codebook of (layer, block, kv = 0, h = 0): [2][Hkv][K][G]
    int B, Hkv, K, Nmax, b0, tok0, ntok;
};

template <typename XT>
__device__ __forceinline__ float ld_xt(const XT *p);
template <>
__device__ __forceinline__ float ld_xt<uint16_t>(const uint16_t *p) { return bf16_to_f32(__ldg(p)); }
template <>
__device__ __forceinline__ float ld_xt<float>(const float *p) { return __ldg(p); }

// Grid: (ntok, Tc, nb); 32 threads.
template <int D, typename XT>
__global__ void __launch_bounds__(32) tasq_sigma_kernel(const TasqArgs a) {
    const int nrel = blockIdx.x, m = blockIdx.y, brel = blockIdx.z;
    const int lane = threadIdx.x;
    const XT *xk = reinterpret_cast<const XT *>(a.xk);
    double ss = 0.0;
    for (int h = 0; h < a.Hkv; ++h) {
        const XT *x = xk + (size_t)m * a.s0 + (size_t)brel * a.s1 + (size_t)nrel * a.s2 + (size_t)h * a.s3;
        const float *w = a.w + ((size_t)m * a.Hkv + h) * D;
#pragma unroll
        for (int f = lane; f < D; f += 32) {
            const double v = __dmul_rn((double)__ldg(w + f), (double)ld_xt(x + f));
            ss = __dadd_rn(ss, __dmul_rn(v, v));
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    if (lane == 0) {
        const double rms = sqrt(ss / ((double)a.Hkv * D));
        a.sigma[((size_t)m * a.B + a.b0 + brel) * a.Nmax + a.tok0 + nrel] = __half_as_ushort(__double2half(rms));
    }
}

// Grid: (ceil(ntok * NP / 128), Hkv, nb); one thread per index word.
template <int D, int C, int TC, typename XT>
__global__ void __launch_bounds__(128) tasq_encode_kernel(const TasqArgs a) {
    constexpr int G = C * TC;
    constexpr int NP = D / (2 * C);
    extern __shared__ __align__(16) float ecb[];           // [2][K][G] fp32, then the permutation
    const int h = blockIdx.y;
    const int brel = blockIdx.z;
    const int b = a.b0 + brel;
    const int K = a.K;
    stage_codebooks<G>(ecb, a.cb, a.Hkv, h, K);
    int16_t *perm = reinterpret_cast<int16_t *>(ecb + 2 * (size_t)K * G);
    for (int j = threadIdx.x; j < D / 2; j += blockDim.x) perm[j] = a.perm[(size_t)h * (D / 2) + j] & (D / 2 - 1);
    __syncthreads();

    const int wl = blockIdx.x * blockDim.x + threadIdx.x;
    if (wl >= a.ntok * NP) return;
    const int nrel = wl / NP;
    const int p = wl % NP;
    const XT *xk = reinterpret_cast<const XT *>(a.xk);
    const XT *xv = reinterpret_cast<const XT *>(a.xv);
    const size_t base = (size_t)brel * a.s1 + (size_t)nrel * a.s2 + (size_t)h * a.s3;
    float z[4][G];
#pragma unroll
    for (int m = 0; m < TC; ++m) {
        const size_t off = base + (size_t)m * a.s0;
        const float *w = a.w + ((size_t)m * a.Hkv + h) * D;
        const float sg = __half2float(__ushort_as_half(a.sigma[((size_t)m * a.B + b) * a.Nmax + a.tok0 + nrel]));
#pragma unroll
        for (int i = 0; i < C; ++i) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {                 // TaSQ groups 2p and 2p + 1
                const int lowf = perm[(2 * p + u) * (C / 2) + i / 2];
                const int f = (i & 1) ? lowf + D / 2 : lowf;
                z[u][i * TC + m] = __fdiv_rn(__fmul_rn(__ldg(w + f), ld_xt(xk + off + f)), sg);
            }
            z[2][i * TC + m] = ld_xt(xv + off + p * C + i);
            z[3][i * TC + m] = ld_xt(xv + off + (p + NP) * C + i);
        }
    }
    const uint32_t word = nearest_word<G>(z, ecb, ecb + (size_t)K * G, K);
    a.idx[((size_t)b * a.Hkv + h) * idx_words_per_bh(a.Nmax, D, C) + idx_word(a.tok0 + nrel, p, NP)] = word;
}

// parts: 1 = the scales, 2 = the CUDA-core encode, 3 = both
template <int D, int C, int TC, typename XT>
static cudaError_t launch_tasq_t(const TasqArgs &a, int nb, int parts, cudaStream_t s) {
    constexpr int NP = D / (2 * C);
    cudaError_t e = cudaSuccess;
    if (parts & 1) {
        tasq_sigma_kernel<D, XT><<<dim3(a.ntok, TC, nb), 32, 0, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (!(parts & 2)) return cudaSuccess;
    const size_t smem = 2 * (size_t)a.K * C * TC * sizeof(float) + (D / 2) * sizeof(int16_t);
    auto k = tasq_encode_kernel<D, C, TC, XT>;
    if ((e = ensure_dynamic_smem((const void *)k, smem)) != cudaSuccess) return e;
    k<<<dim3((a.ntok * NP + 127) / 128, a.Hkv, nb), 128, smem, s>>>(a);
    return cudaGetLastError();
}

template <int D, typename XT>
static cudaError_t dispatch_tasq(int c, int tc, const TasqArgs &a, int nb, int parts, cudaStream_t s) {
    if (c == 4 && tc == 4) return launch_tasq_t<D, 4, 4, XT>(a, nb, parts, s);
    if (c == 4 && tc == 2) return launch_tasq_t<D, 4, 2, XT>(a, nb, parts, s);
    if (c == 4 && tc == 1) return launch_tasq_t<D, 4, 1, XT>(a, nb, parts, s);
    if (c == 8 && tc == 4) return launch_tasq_t<D, 8, 4, XT>(a, nb, parts, s);
    if (c == 8 && tc == 2) return launch_tasq_t<D, 8, 2, XT>(a, nb, parts, s);
    if (c == 8 && tc == 1) return launch_tasq_t<D, 8, 1, XT>(a, nb, parts, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_tasq_encode(const loopvq_cache &cc, const loopvq_tasq &tq, int layer, int block, const void *xk,
                               const void *xv, int x_dtype, const int64_t *strides, int b0, int nb, int tok0, int ntok,
                               cudaStream_t s) {
    if (nb == 0 || ntok == 0) return cudaSuccess;
    const int NB = cc.T / cc.Tc;
    const int t0 = block * cc.Tc;
    TasqArgs a{};
    a.xk = xk;
    a.xv = xv;
    a.s0 = strides[0];
    a.s1 = strides[1];
    a.s2 = strides[2];
    a.s3 = strides[3];
    a.w = tq.w + ((size_t)layer * cc.T + t0) * cc.Hkv * cc.D;
    a.perm = tq.perm + ((size_t)layer * NB + block) * cc.Hkv * (cc.D / 2);
    a.sigma = tq.sigma + ((size_t)layer * cc.T + t0) * cc.B * cc.Nmax;
    a.idx = cc.idx + idx_base(cc, layer, block, 0, 0);
    a.cb = cc.codebook + codebook_base(cc, layer, block, 0, 0);
    a.B = cc.B;
    a.Hkv = cc.Hkv;
    a.K = cc.K;
    a.Nmax = cc.Nmax;
    a.b0 = b0;
    a.tok0 = tok0;
    a.ntok = ntok;
    const bool bf = x_dtype == LOOPVQ_BF16;
    auto run = [&](int parts) -> cudaError_t {
        if (cc.D == 128)
            return bf ? dispatch_tasq<128, uint16_t>(cc.c, cc.Tc, a, nb, parts, s)
                      : dispatch_tasq<128, float>(cc.c, cc.Tc, a, nb, parts, s);
        if (cc.D == 64)
            return bf ? dispatch_tasq<64, uint16_t>(cc.c, cc.Tc, a, nb, parts, s)
                      : dispatch_tasq<64, float>(cc.c, cc.Tc, a, nb, parts, s);
        return cudaErrorInvalidValue;
    };
    if (!bf) return run(3);
    // bf16 keys and values: the scales, then the tensor-core encode where the shape has one
    cudaError_t e = run(1);
    if (e != cudaSuccess) return e;
    e = launch_tasq_encode_tc(cc, tq, layer, block, xk, xv, strides, b0, nb, tok0, ntok, s);
    if (e != cudaErrorNotSupported) return e;
    return run(2);
}

}  // namespace loopvq
