// Load-time preparation: per-loop-step codebook slices and the RoPE table.
//
// Slice of loop step t = beta*Tc + m keeps coordinates i*Tc + m (i < c) of every
// entry of the block's codebook (LoopVQ paper, Sec. 4.3 "Attention": B_t, cut once
// when the model is loaded; Sec. 4.1 eq. (5)).  The RoPE table holds cos and sin
// of the D/2 frequencies at every position, one row per position (App. C), with
// angles formed in fp64 so positions up to 32K keep full fp32 accuracy.
#include "loopvq_internal.cuh"

namespace loopvq {

__global__ void slice_cut_kernel(const uint16_t *__restrict__ cb, uint16_t *__restrict__ slices,
                                 int L, int T, int Tc, int Hkv, int K, int c, int ncb, size_t total) {
    const int G = c * Tc;
    const int NB = T / Tc;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        // e enumerates [L][T][2][Hkv][K][ncb][c]: row r of a slice holds entry r of every codebook
        size_t r0 = e;
        const int i = (int)(r0 % c); r0 /= c;
        const int g = (int)(r0 % ncb); r0 /= ncb;
        const int r = (int)(r0 % K); r0 /= K;
        const int h = (int)(r0 % Hkv); r0 /= Hkv;
        const int kv = (int)(r0 % 2); r0 /= 2;
        const int t = (int)(r0 % T); r0 /= T;
        const int layer = (int)r0;
        const int beta = t / Tc, m = t % Tc;
        const size_t src = (((((size_t)layer * NB + beta) * 2 + kv) * Hkv + h) * ncb + g) * (size_t)K * G +
                           (size_t)r * G + (size_t)i * Tc + m;
        slices[e] = cb[src];
    }
}

__global__ void rope_table_kernel(float *__restrict__ rope, int Nmax, int D, double theta) {
    const int h = D / 2;
    const size_t total = (size_t)Nmax * h;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const int f = (int)(e % h);
        const int p = (int)(e / h);
        const double omega = pow(theta, -2.0 * (double)f / (double)D);
        const double ang = (double)p * omega;
        double sn, cs;
        sincos(ang, &sn, &cs);
        rope[(size_t)p * D + f] = (float)cs;
        rope[(size_t)p * D + h + f] = (float)sn;
    }
}

cudaError_t launch_prepare(const loopvq_cache &cc, cudaStream_t s) {
    const size_t ns = (size_t)cc.L * cc.T * 2 * cc.Hkv * cc.K * cc.c * ncb_of(cc);
    int blocks = (int)((ns + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    slice_cut_kernel<<<blocks, 256, 0, s>>>(cc.codebook, cc.slices, cc.L, cc.T, cc.Tc, cc.Hkv, cc.K, cc.c, ncb_of(cc),
                                            ns);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t nr = (size_t)cc.Nmax * (cc.D / 2);
    blocks = (int)((nr + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    rope_table_kernel<<<blocks, 256, 0, s>>>(cc.rope, cc.Nmax, cc.D, (double)cc.theta);
    return cudaGetLastError();
}

// Explicit reconstruction of loop step t for one sequence (eq. 5), optionally
// rotated by RoPE at each token's position (keys only).  One thread per
// (head, token, frequency f < D/2) writes channels f and f + D/2.
__global__ void dequant_kernel(loopvq_cache cc, int layer, int t, int kv, int b, int tok0, int ntok,
                               int apply_rope, float *__restrict__ out) {
    const int D = cc.D, c = cc.c, h2 = D / 2, NP = D / (2 * c);
    const int beta = t / cc.Tc;
    const size_t total = (size_t)cc.Hkv * ntok * h2;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const int f = (int)(e % h2);
        const int n = (int)((e / h2) % ntok);
        const int h = (int)(e / ((size_t)h2 * ntok));
        const int tok = tok0 + n;
        const int p = f / c, i = f % c;          // pair-group and channel within the group
        const uint32_t w = cc.idx[idx_base(cc, layer, beta, b, h) + idx_word(tok, p, NP)];
        const int r_lo = (w >> (16 * kv)) & 0xff;
        const int r_hi = (w >> (16 * kv + 8)) & 0xff;
        const uint16_t *S = cc.slices + slice_base(cc, layer, t, kv, h);
        // row r of the slice holds entry r of every codebook: NCB * c values; a shared codebook's entry
        // is the whole row, a per-group codebook's entry for group g sits at g * c
        const int rs = ncb_of(cc) * c;
        const int glo = ncb_of(cc) > 1 ? p * c : 0, ghi = ncb_of(cc) > 1 ? (p + NP) * c : 0;
        // codes outside [0, K) rebuild as zero, like the zeroed rows of the decode kernel
        float lo = r_lo < cc.K ? bf16_to_f32(S[(size_t)r_lo * rs + glo + i]) : 0.f;
        float hi = r_hi < cc.K ? bf16_to_f32(S[(size_t)r_hi * rs + ghi + i]) : 0.f;
        if (apply_rope && kv == 0) {
            const float cs = cc.rope[(size_t)tok * D + f];
            const float sn = cc.rope[(size_t)tok * D + h2 + f];
            const float a = lo, bb = hi;
            lo = a * cs - bb * sn;
            hi = bb * cs + a * sn;
        }
        float *o = out + ((size_t)h * ntok + n) * D;
        o[f] = lo;
        o[h2 + f] = hi;
    }
}

cudaError_t launch_dequant(const loopvq_cache &cc, int layer, int t, int kv, int b, int tok0, int ntok,
                           int apply_rope, float *out, cudaStream_t s) {
    const size_t total = (size_t)cc.Hkv * ntok * (cc.D / 2);
    if (total == 0) return cudaSuccess;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    dequant_kernel<<<blocks, 256, 0, s>>>(cc, layer, t, kv, b, tok0, ntok, apply_rope, out);
    return cudaGetLastError();
}

}  // namespace loopvq
