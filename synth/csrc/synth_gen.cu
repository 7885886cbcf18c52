// Bulk generation of the seeded synthetic workloads on the GPU.
//
// Same definitions as synth/philox.py and synth/workloads.py, bit for bit:
// Philox4x32-10 (Salmon et al., SC'11) keyed by (seed, 0x4C565142) on the counter
// (flat_lo, flat_hi, step, tag << 24 | layer); an approx-normal is the centred
// Irwin-Hall sum of the eight 16-bit halves of one Philox block times one fp32
// constant; loop-axis AR(1) in fp32 with separately rounded multiply, multiply,
// add; bf16 by round-to-nearest-even.  Generation only: nothing of the
// quantisation method is computed here.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u, kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
constexpr uint32_t kKey1 = 0x4C565142u;
constexpr int kMaxSteps = 64;

struct Coef {
    float rho[kMaxSteps];
    float sig[kMaxSteps];
};

__device__ __forceinline__ uint4 philox(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(kM0, c.x), lo0 = kM0 * c.x;
        const uint32_t hi1 = __umulhi(kM1, c.z), lo1 = kM1 * c.z;
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += kW0;
        k1 += kW1;
    }
    return c;
}

__device__ __forceinline__ float approx_normal(uint64_t flat, uint32_t step, uint32_t tagl, uint32_t seed,
                                               float ih_scale) {
    const uint4 w = philox(make_uint4((uint32_t)flat, (uint32_t)(flat >> 32), step, tagl), seed, kKey1);
    const int s = (int)(w.x & 0xffff) + (int)(w.x >> 16) + (int)(w.y & 0xffff) + (int)(w.y >> 16) +
                  (int)(w.z & 0xffff) + (int)(w.z >> 16) + (int)(w.w & 0xffff) + (int)(w.w >> 16);
    return __fmul_rn((float)(s - 262140), ih_scale);
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// K or V cache: out [t_last - t_first + 1][B][Nmax][H][D] bf16, AR(1) over loops 0..t_last.
__global__ void kv_kernel(uint16_t *out, uint32_t seed, uint32_t tagl, int t_first, int t_last, int B, int Nmax,
                          int H, int D, Coef cf, float ih_scale) {
    const size_t per_t = (size_t)B * Nmax * H * D;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < per_t; e += (size_t)gridDim.x * blockDim.x) {
        float x = 0.f;
        for (int t = 0; t <= t_last; ++t) {
            const float n = approx_normal(e, (uint32_t)t, tagl, seed, ih_scale);
            x = t == 0 ? n : __fadd_rn(__fmul_rn(cf.rho[t], x), __fmul_rn(cf.sig[t], n));
            if (t >= t_first) out[(size_t)(t - t_first) * per_t + e] = bf16_bits(x);
        }
    }
}

// Queries [B][Hq][D] bf16 of one (layer, loop step).
__global__ void q_kernel(uint16_t *out, uint32_t seed, uint32_t tagl, int step, size_t n, float ih_scale, float gain) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        float x = approx_normal(e, (uint32_t)step, tagl, seed, ih_scale);
        if (gain != 1.f) x = __fmul_rn(x, gain);
        out[e] = bf16_bits(x);
    }
}

// Codebooks of every (layer, block, kv, head, group) in the [L][NB][2][Hkv][NCB][K][G] order.
__global__ void codebook_kernel(uint16_t *out, uint32_t seed, int L, int NB, int Tc, int Hkv, int NCB, int K, int c,
                                Coef cf, float ih_scale, uint32_t tag_k, uint32_t tag_v) {
    const int G = c * Tc;
    const size_t total = (size_t)L * NB * 2 * Hkv * NCB * K * c;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        size_t r0 = e;
        const int i = (int)(r0 % c); r0 /= c;
        const int r = (int)(r0 % K); r0 /= K;
        const int g = (int)(r0 % NCB); r0 /= NCB;
        const int h = (int)(r0 % Hkv); r0 /= Hkv;
        const int kv = (int)(r0 % 2); r0 /= 2;
        const int blk = (int)(r0 % NB); r0 /= NB;
        const int layer = (int)r0;
        const uint64_t flat = (((uint64_t)h * NCB + g) * K + r) * c + i;
        const uint32_t tagl = ((kv ? tag_v : tag_k) << 24) | (uint32_t)layer;
        const size_t base =
            (((((size_t)layer * NB + blk) * 2 + kv) * Hkv + h) * NCB + g) * (size_t)K * G + (size_t)r * G;
        float x = 0.f;
        for (int m = 0; m < Tc; ++m) {
            const int t = blk * Tc + m;
            const float n = approx_normal(flat, (uint32_t)t, tagl, seed, ih_scale);
            x = m == 0 ? n : __fadd_rn(__fmul_rn(cf.rho[t], x), __fmul_rn(cf.sig[t], n));
            out[base + (size_t)i * Tc + m] = bf16_bits(x);
        }
    }
}

// Uniform random codes packed as index words of one (layer, block) into the tiled word layout
// [B][Hkv][Nmax/4][NP][4]; byte order {K p, K p+NP, V p, V p+NP}.
__global__ void idx_kernel(uint32_t *out, uint32_t seed, uint32_t tagl, int block, int B, int Hkv, int Nmax, int NP,
                           int K) {
    const int ng = 2 * NP;
    const size_t total = (size_t)B * Hkv * Nmax * NP;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        // e enumerates the output words in memory order
        const int k4 = (int)(e & 3);
        size_t r0 = e >> 2;
        const int p = (int)(r0 % NP); r0 /= NP;
        const int tile = (int)(r0 % (Nmax / 4)); r0 /= (Nmax / 4);
        const int h = (int)(r0 % Hkv);
        const int b = (int)(r0 / Hkv);
        const int tok = tile * 4 + k4;
        uint32_t word = 0;
        for (int q = 0; q < 4; ++q) {
            const int kv = q >> 1;
            const int gi = p + (q & 1) * NP;
            const uint64_t flat = (((uint64_t)b * Hkv + h) * Nmax + tok) * ng + gi;
            const uint4 w = philox(make_uint4((uint32_t)flat, (uint32_t)(flat >> 32), (uint32_t)(block * 2 + kv), tagl),
                                   seed, kKey1);
            word |= (w.x % (uint32_t)K) << (8 * q);
        }
        out[e] = word;
    }
}

int grid_for(size_t n) {
    size_t g = (n + 255) / 256;
    return (int)(g > 148 * 64 ? 148 * 64 : (g == 0 ? 1 : g));
}

Coef make_coef(const float *rho, const float *sig, int n) {
    Coef cf{};
    for (int i = 0; i < n && i < kMaxSteps; ++i) {
        cf.rho[i] = rho[i];
        cf.sig[i] = sig[i];
    }
    return cf;
}

}  // namespace

extern "C" {

// rho / sig: host fp32 arrays of t_last + 1 loop coefficients.
int synth_kv(void *out, uint32_t seed, uint32_t tagl, int t_first, int t_last, int B, int Nmax, int H, int D,
             const float *rho, const float *sig, float ih_scale, void *stream) {
    if (t_last >= kMaxSteps || t_first < 0 || t_first > t_last) return 1;
    const size_t n = (size_t)B * Nmax * H * D;
    kv_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t *)out, seed, tagl, t_first, t_last, B, Nmax,
                                                              H, D, make_coef(rho, sig, t_last + 1), ih_scale);
    return (int)cudaGetLastError();
}

int synth_q(void *out, uint32_t seed, uint32_t tagl, int step, size_t n, float ih_scale, float gain, void *stream) {
    q_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t *)out, seed, tagl, step, n, ih_scale, gain);
    return (int)cudaGetLastError();
}

int synth_codebook(void *out, uint32_t seed, int L, int NB, int Tc, int Hkv, int NCB, int K, int c, const float *rho,
                   const float *sig, float ih_scale, uint32_t tag_k, uint32_t tag_v, void *stream) {
    if (NB * Tc > kMaxSteps) return 1;
    const size_t n = (size_t)L * NB * 2 * Hkv * NCB * K * c;
    codebook_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t *)out, seed, L, NB, Tc, Hkv, NCB, K, c,
                                                                    make_coef(rho, sig, NB * Tc), ih_scale, tag_k,
                                                                    tag_v);
    return (int)cudaGetLastError();
}

int synth_idx(void *out, uint32_t seed, uint32_t tagl, int block, int B, int Hkv, int Nmax, int NP, int K,
              void *stream) {
    const size_t n = (size_t)B * Hkv * Nmax * NP;
    idx_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint32_t *)out, seed, tagl, block, B, Hkv, Nmax, NP,
                                                               K);
    return (int)cudaGetLastError();
}

}  // extern "C"
