/*
 * loopvq_oracle.c -- CPU checker for the LoopVQ encode / decode-attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library, and the CUDA library never
 * calls it.
 *
 * It states what the method computes in the most direct way: plain loops, one
 * element at a time, in the order the definitions are written.
 *
 *   encode     nearest codebook entry of each coupled sub-vector, squared
 *              distance accumulated in fp32 over the coordinates in ascending
 *              order, first (lowest) index kept on ties.
 *              LoopVQ paper, Sec. 2 "Vector quantization of the KV cache",
 *              eq. (2); Sec. 4.1 "Loop-axis vector quantization", eq. (4).
 *   dequant    loop step m of a block copies coordinate i*Tc + m of the
 *              selected entry into channel g*c + i, for i < c.
 *              LoopVQ paper, Sec. 4.1 eq. (5); Sec. 4.3 "Attention"; App. A.2.
 *   rope       half-split rotary embedding in fp64 applied to reconstructed
 *              keys only, pairs (f, f + D/2), angle p * theta^(-2f/D).
 *              LoopVQ paper, Sec. 2 (keys quantized before RoPE); App. C.
 *   attention  softmax attention of one query over the reconstructed cache in
 *              fp64, two passes (max, then sum); lse = max + ln(sum).
 *              LoopVQ paper, Sec. 4.3 "Attention".
 *   splits     the same attention computed per split of the tokens and merged
 *              through the log-sum-exp of each split (Flash-Decoding merge),
 *              which the pages state recovers the exact softmax.
 *              LoopVQ paper, Sec. 4.3 "Attention".
 *   *_pg       the same with one codebook per channel group, E_g for group g
 *              (the paper's notation B_{beta,l,h,g}): encode, the distance
 *              check, reconstruction and decode.
 *              LoopVQ paper, Sec. 2 eq. (2); Sec. 4.1 eq. (5); App. A.2.
 *   tasq_*     TaSQ applied before loop-axis coupling: u = P(w (.) k / sigma),
 *              with w a per-channel weight, sigma the root mean square of
 *              w (.) k over all heads and channels of the token (stored in
 *              fp16), and P a permutation that keeps every RoPE pair
 *              {f, f + D/2} inside one code; the coupled key vectors are built
 *              from u, reconstruction inverts the transform before RoPE.
 *              LoopVQ paper, App. B "Formulation", "Grouping under loop
 *              coupling", "Calibration and bitwidth".
 *   windowed   attention of one query over a cache whose sink and recent
 *              tokens are kept in bf16 (keys stored already rotated) and whose
 *              other tokens lo <= n < hi are coded: the coded keys are rebuilt
 *              and rotated at their absolute positions, all keys are put in
 *              one list, and one softmax runs over the list.
 *              LoopVQ paper, Sec. 4.3 "Cache layout" and "Attention".
 *
 * Array conventions (all dense, row-major, caller-owned):
 *   x   float  [Tc][N][D]   one block of Tc loop steps of one (layer, head, K|V)
 *   E   float  [K][G]       codebook, G = c*Tc, coordinate i*Tc + m
 *   idx uint8  [N][D/c]     code of channel group g (channels g*c .. g*c+c-1)
 *   q   double [D]          query, already rotated at its own position
 * Inputs that are bf16 in the method are passed as the exactly widened floats.
 *
 * Parity pins live in tests/test_oracle_pins.py; every function here is pinned
 * there by a check that does not re-use this file's arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/* Coupled vector of token n, channel group g (eq. 4):
 *   z[i*Tc + m] = x[m][n][g*c + i],  i < c, m < Tc. */
static void coupled_vector(const float *x, int Tc, int N, int D, int c, int n, int g, float *z)
{
    for (int i = 0; i < c; ++i)
        for (int m = 0; m < Tc; ++m)
            z[i * Tc + m] = x[((size_t)m * N + n) * D + (size_t)g * c + i];
}

/* Nearest entry (eq. 2) of every coupled vector; fp32 distances, lowest index on ties. */
void ora_encode(const float *x, int Tc, int N, int D, int c, const float *E, int K, uint8_t *idx)
{
    const int G = c * Tc;
    const int ng = D / c;
    float z[256];
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < ng; ++g) {
            coupled_vector(x, Tc, N, D, c, n, g, z);
            int best = 0;
            float best_d = INFINITY;
            for (int r = 0; r < K; ++r) {
                float d = 0.0f;
                for (int k = 0; k < G; ++k) {
                    float diff = z[k] - E[(size_t)r * G + k];
                    float sq = diff * diff;
                    d = d + sq;
                }
                if (d < best_d) { best_d = d; best = r; }
            }
            idx[(size_t)n * ng + g] = (uint8_t)best;
        }
    }
}

/* fp64 squared distance between coupled vector (n, g) and entry r; used to classify near-ties. */
double ora_dist64(const float *x, int Tc, int N, int D, int c, const float *E, int n, int g, int r)
{
    const int G = c * Tc;
    float z[256];
    coupled_vector(x, Tc, N, D, c, n, g, z);
    double d = 0.0;
    for (int k = 0; k < G; ++k) {
        double diff = (double)z[k] - (double)E[(size_t)r * G + k];
        d += diff * diff;
    }
    return d;
}

/* Reconstruction of loop step m of the block (eq. 5): out[n][g*c + i] = E[idx[n][g]][i*Tc + m]. */
void ora_dequant(const uint8_t *idx, int N, int D, int c, int Tc, int m, const float *E, double *out)
{
    const int G = c * Tc;
    const int ng = D / c;
    for (int n = 0; n < N; ++n)
        for (int g = 0; g < ng; ++g) {
            int r = idx[(size_t)n * ng + g];
            for (int i = 0; i < c; ++i)
                out[(size_t)n * D + (size_t)g * c + i] = (double)E[(size_t)r * G + i * Tc + m];
        }
}

/* Half-split RoPE in fp64 at positions pos0 + n (App. C; pairs (f, f + D/2)). */
void ora_rope(double *x, int N, int D, double theta, int pos0)
{
    const int h = D / 2;
    for (int n = 0; n < N; ++n) {
        double p = (double)(pos0 + n);
        for (int f = 0; f < h; ++f) {
            double omega = pow(theta, -2.0 * (double)f / (double)D);
            double ang = p * omega;
            double cs = cos(ang), sn = sin(ang);
            double a = x[(size_t)n * D + f];
            double b = x[(size_t)n * D + f + h];
            x[(size_t)n * D + f] = a * cs - b * sn;
            x[(size_t)n * D + f + h] = b * cs + a * sn;
        }
    }
}

/* Softmax attention of q over N keys/values in fp64, two passes.  N == 0 gives out = 0, lse = -inf. */
void ora_attention(const double *q, const double *k, const double *v, int N, int D, double scale,
                   double *out, double *lse)
{
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (N <= 0) { *lse = -INFINITY; return; }
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double mx = -INFINITY;
    for (int n = 0; n < N; ++n) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * k[(size_t)n * D + d];
        s[n] = dot * scale;
        if (s[n] > mx) mx = s[n];
    }
    double sum = 0.0;
    for (int n = 0; n < N; ++n) {
        double p = exp(s[n] - mx);
        sum += p;
        for (int d = 0; d < D; ++d) out[d] += p * v[(size_t)n * D + d];
    }
    for (int d = 0; d < D; ++d) out[d] /= sum;
    *lse = mx + log(sum);
    free(s);
}

/* The same attention split at bounds[0] = 0 < ... < bounds[nsplit] = N: each split is attended on its
 * own, giving (out_s, lse_s); the splits are merged by weights exp(lse_s - max_s lse_s). */
void ora_attention_splits(const double *q, const double *k, const double *v, int N, int D, double scale,
                          const int *bounds, int nsplit, double *out, double *lse)
{
    double *os = (double *)malloc(sizeof(double) * (size_t)D * (size_t)(nsplit > 0 ? nsplit : 1));
    double *ls = (double *)malloc(sizeof(double) * (size_t)(nsplit > 0 ? nsplit : 1));
    double mx = -INFINITY;
    for (int s = 0; s < nsplit; ++s) {
        int a = bounds[s], b = bounds[s + 1];
        ora_attention(q, k + (size_t)a * D, v + (size_t)a * D, b - a, D, scale, os + (size_t)s * D, &ls[s]);
        if (ls[s] > mx) mx = ls[s];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (mx == -INFINITY) { *lse = -INFINITY; free(os); free(ls); return; }
    double wsum = 0.0;
    for (int s = 0; s < nsplit; ++s) {
        if (ls[s] == -INFINITY) continue;
        double w = exp(ls[s] - mx);
        wsum += w;
        for (int d = 0; d < D; ++d) out[d] += w * os[(size_t)s * D + d];
    }
    for (int d = 0; d < D; ++d) out[d] /= wsum;
    *lse = mx + log(wsum);
    free(os);
    free(ls);
}

/* Decode attention of one query at loop step m of a block over a coded cache of N tokens
 * (Sec. 4.3): reconstruct keys (eq. 5), rotate them at positions 0..N-1, reconstruct values,
 * attend.  Scratch is allocated here; the checker is not a hot path. */
void ora_decode(const double *q, const uint8_t *idx_k, const uint8_t *idx_v, const float *E_k,
                const float *E_v, int N, int D, int c, int Tc, int m, double theta, double scale,
                double *out, double *lse)
{
    size_t nd = (size_t)(N > 0 ? N : 1) * (size_t)D;
    double *kh = (double *)malloc(sizeof(double) * nd);
    double *vh = (double *)malloc(sizeof(double) * nd);
    ora_dequant(idx_k, N, D, c, Tc, m, E_k, kh);
    ora_rope(kh, N, D, theta, 0);
    ora_dequant(idx_v, N, D, c, Tc, m, E_v, vh);
    ora_attention(q, kh, vh, N, D, scale, out, lse);
    free(kh);
    free(vh);
}

/* Attention of one query over NW bf16 window tokens (keys kw already rotated, values vw, both
 * [NW][D]) together with the coded tokens lo <= n < hi, whose codes are rows 0 .. hi-lo-1 of
 * idx_k / idx_v (Sec. 4.3 "Cache layout": sink and recent tokens in bf16, the rest coded).  The
 * coded keys are rebuilt (eq. 5) and rotated at positions lo .. hi-1; then one softmax runs over the
 * concatenated key list: window tokens first, coded tokens after. */
void ora_decode_windowed(const double *q, const double *kw, const double *vw, int NW, const uint8_t *idx_k,
                         const uint8_t *idx_v, const float *E_k, const float *E_v, int lo, int hi, int D, int c,
                         int Tc, int m, double theta, double scale, double *out, double *lse)
{
    const int NC = hi > lo ? hi - lo : 0;
    const int N = NW + NC;
    size_t nd = (size_t)(N > 0 ? N : 1) * (size_t)D;
    double *kh = (double *)malloc(sizeof(double) * nd);
    double *vh = (double *)malloc(sizeof(double) * nd);
    for (size_t i = 0; i < (size_t)NW * D; ++i) {
        kh[i] = kw[i];
        vh[i] = vw[i];
    }
    double *kc = kh + (size_t)NW * D, *vc = vh + (size_t)NW * D;
    ora_dequant(idx_k, NC, D, c, Tc, m, E_k, kc);
    ora_rope(kc, NC, D, theta, lo);
    ora_dequant(idx_v, NC, D, c, Tc, m, E_v, vc);
    ora_attention(q, kh, vh, N, D, scale, out, lse);
    free(kh);
    free(vh);
}

/* ---- one codebook per channel group: E holds ng = D/c codebooks [ng][K][G], group g uses E_g ---- */

/* Nearest entry of every coupled vector in its own group's codebook; fp32, lowest index on ties. */
void ora_encode_pg(const float *x, int Tc, int N, int D, int c, const float *E, int K, uint8_t *idx)
{
    const int G = c * Tc;
    const int ng = D / c;
    float z[256];
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < ng; ++g) {
            const float *Eg = E + (size_t)g * K * G;
            coupled_vector(x, Tc, N, D, c, n, g, z);
            int best = 0;
            float best_d = INFINITY;
            for (int r = 0; r < K; ++r) {
                float d = 0.0f;
                for (int k = 0; k < G; ++k) {
                    float diff = z[k] - Eg[(size_t)r * G + k];
                    float sq = diff * diff;
                    d = d + sq;
                }
                if (d < best_d) { best_d = d; best = r; }
            }
            idx[(size_t)n * ng + g] = (uint8_t)best;
        }
    }
}

double ora_dist64_pg(const float *x, int Tc, int N, int D, int c, const float *E, int K, int n, int g, int r)
{
    return ora_dist64(x, Tc, N, D, c, E + (size_t)g * K * c * Tc, n, g, r);
}

/* Reconstruction of loop step m with per-group codebooks: out[n][g*c + i] = E_g[idx[n][g]][i*Tc + m]. */
void ora_dequant_pg(const uint8_t *idx, int N, int D, int c, int Tc, int m, const float *E, int K, double *out)
{
    const int G = c * Tc;
    const int ng = D / c;
    for (int n = 0; n < N; ++n)
        for (int g = 0; g < ng; ++g) {
            const float *Eg = E + (size_t)g * K * G;
            int r = idx[(size_t)n * ng + g];
            for (int i = 0; i < c; ++i)
                out[(size_t)n * D + (size_t)g * c + i] = (double)Eg[(size_t)r * G + i * Tc + m];
        }
}

/* Decode attention as ora_decode, with per-group codebooks for keys and values. */
void ora_decode_pg(const double *q, const uint8_t *idx_k, const uint8_t *idx_v, const float *E_k,
                   const float *E_v, int K, int N, int D, int c, int Tc, int m, double theta, double scale,
                   double *out, double *lse)
{
    size_t nd = (size_t)(N > 0 ? N : 1) * (size_t)D;
    double *kh = (double *)malloc(sizeof(double) * nd);
    double *vh = (double *)malloc(sizeof(double) * nd);
    ora_dequant_pg(idx_k, N, D, c, Tc, m, E_k, K, kh);
    ora_rope(kh, N, D, theta, 0);
    ora_dequant_pg(idx_v, N, D, c, Tc, m, E_v, K, vh);
    ora_attention(q, kh, vh, N, D, scale, out, lse);
    free(kh);
    free(vh);
}

/* ---- TaSQ before loop-axis coupling (App. B) ---- */

/* Round to the nearest fp16 value, ties to even (IEEE 754 binary16: 1 sign, 5 exponent bits with
 * bias 15, 10 fraction bits; subnormals below 2^-14; overflow to infinity), returned as a double. */
double ora_round_fp16(double x)
{
    if (x != x) return x;
    const double ax = fabs(x);
    if (ax >= 65520.0) return x < 0 ? -INFINITY : INFINITY;     /* 65504 + half an ulp rounds up */
    int e;
    frexp(ax, &e);                                               /* ax = f * 2^e, f in [0.5, 1) */
    int exp2 = e - 1;                                            /* ax in [2^exp2, 2^(exp2+1)) */
    if (exp2 < -14) exp2 = -14;                                  /* subnormal spacing 2^-24 */
    const double ulp = ldexp(1.0, exp2 - 10);
    const double q = ax / ulp;                                   /* exact: a power-of-two scaling */
    double r = floor(q);
    const double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    const double y = r * ulp;
    return x < 0 ? -y : y;
}

/* sigma of every token for one (loop step, layer, sequence): the root mean square of w (.) k over all
 * Hkv heads and D channels, in fp64, rounded to fp16.  k: [Hkv][N][D], w: [Hkv][D]. */
void ora_tasq_sigma(const float *k, const float *w, int Hkv, int N, int D, double *sigma)
{
    for (int n = 0; n < N; ++n) {
        double ss = 0.0;
        for (int h = 0; h < Hkv; ++h)
            for (int f = 0; f < D; ++f) {
                const double v = (double)w[(size_t)h * D + f] * (double)k[((size_t)h * N + n) * D + f];
                ss += v * v;
            }
        sigma[n] = ora_round_fp16(sqrt(ss / ((double)Hkv * D)));
    }
}

/* Channel of coordinate i < c of TaSQ group g: the group holds the c/2 RoPE pairs whose low
 * channels are perm[g*c/2 + j], j < c/2, each pair as (low, low + D/2). */
static int tasq_channel(const int16_t *perm, int D, int c, int g, int i)
{
    const int f = perm[g * (c / 2) + i / 2];
    return (i % 2) ? f + D / 2 : f;
}

/* u = (w (.) k) / sigma of every token, in fp32 (multiply then divide, each rounded).
 * k: [N][D] of one loop step, w: [D], sigma: [N] (fp16 values); u: [N][D]. */
void ora_tasq_transform(const float *k, const float *w, const double *sigma, int N, int D, float *u)
{
    for (int n = 0; n < N; ++n)
        for (int f = 0; f < D; ++f) {
            const float wk = w[f] * k[(size_t)n * D + f];
            u[(size_t)n * D + f] = wk / (float)sigma[n];
        }
}

/* TaSQ + LoopVQ encode of one (layer, block, head) (App. B eq. 11): coupled vector of group g is
 * z[i*Tc + m] = u^(m)[channel(g, i)]; nearest entry in fp32 as ora_encode.
 * x: [Tc][N][D] keys, w: [Tc][D], sigma: [Tc][N], perm: [D/2]; idx: [N][D/c]. */
void ora_tasq_encode(const float *x, const float *w, const double *sigma, const int16_t *perm, int Tc, int N, int D,
                     int c, const float *E, int K, uint8_t *idx)
{
    const int G = c * Tc;
    const int ng = D / c;
    float *u = (float *)malloc(sizeof(float) * (size_t)Tc * (N > 0 ? N : 1) * D);
    for (int m = 0; m < Tc; ++m)
        ora_tasq_transform(x + (size_t)m * N * D, w + (size_t)m * D, sigma + (size_t)m * N, N, D,
                           u + (size_t)m * N * D);
    float z[256];
    for (int n = 0; n < N; ++n)
        for (int g = 0; g < ng; ++g) {
            for (int i = 0; i < c; ++i)
                for (int m = 0; m < Tc; ++m)
                    z[i * Tc + m] = u[((size_t)m * N + n) * D + tasq_channel(perm, D, c, g, i)];
            int best = 0;
            float best_d = INFINITY;
            for (int r = 0; r < K; ++r) {
                float d = 0.0f;
                for (int k = 0; k < G; ++k) {
                    float diff = z[k] - E[(size_t)r * G + k];
                    float sq = diff * diff;
                    d = d + sq;
                }
                if (d < best_d) { best_d = d; best = r; }
            }
            idx[(size_t)n * ng + g] = (uint8_t)best;
        }
    free(u);
}

/* Reconstruction of the keys at loop step m (the transform inverted, fp64):
 * k_hat[n][channel(g, i)] = sigma[n] * E[idx[n][g]][i*Tc + m] / w[channel(g, i)].
 * w: [D] of that loop step, sigma: [N] of that loop step. */
void ora_tasq_dequant(const uint8_t *idx, int N, int D, int c, int Tc, int m, const float *E, const int16_t *perm,
                      const float *w, const double *sigma, double *out)
{
    const int G = c * Tc;
    const int ng = D / c;
    for (int n = 0; n < N; ++n)
        for (int g = 0; g < ng; ++g) {
            const int r = idx[(size_t)n * ng + g];
            for (int i = 0; i < c; ++i) {
                const int f = tasq_channel(perm, D, c, g, i);
                out[(size_t)n * D + f] = sigma[n] * (double)E[(size_t)r * G + i * Tc + m] / (double)w[f];
            }
        }
}

/* Decode attention with TaSQ keys: keys rebuilt by ora_tasq_dequant and rotated at positions 0..N-1,
 * values rebuilt as in ora_decode (values are not transformed). */
void ora_tasq_decode(const double *q, const uint8_t *idx_k, const uint8_t *idx_v, const float *E_k, const float *E_v,
                     const int16_t *perm, const float *w, const double *sigma, int N, int D, int c, int Tc, int m,
                     double theta, double scale, double *out, double *lse)
{
    size_t nd = (size_t)(N > 0 ? N : 1) * (size_t)D;
    double *kh = (double *)malloc(sizeof(double) * nd);
    double *vh = (double *)malloc(sizeof(double) * nd);
    ora_tasq_dequant(idx_k, N, D, c, Tc, m, E_k, perm, w, sigma, kh);
    ora_rope(kh, N, D, theta, 0);
    ora_dequant(idx_v, N, D, c, Tc, m, E_v, vh);
    ora_attention(q, kh, vh, N, D, scale, out, lse);
    free(kh);
    free(vh);
}
