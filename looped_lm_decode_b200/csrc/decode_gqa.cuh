// Split-K decode attention over the loop-axis coded cache, 4 query heads per KV head, D = 128,
// channel groups of 8 (the quarter-bit grouped-query workload): the rebuilt key is rotated once and
// scored against the 4 heads on CUDA cores, and the values of all 4 heads accumulate on the tensor
// cores.
//
// LoopVQ paper, Sec. 4.3 "Attention" and App. C: every index is looked up in the loop step's codebook
// slice held in shared memory, keys are rebuilt before RoPE and rotated at their positions, and the
// tokens are cut into splits whose partial outputs are merged through their log-sum-exp.
//
// Design (B200, sm_100a):
//  * The tile space, pieces, partial records and merge are those of decode_split_kernel
//    (decode_kernel.cuh, decode_merge.cuh).  The slices are staged as bank-private replicas: the K entry converted to
//    fp32 (32 bytes) with its two halves in 8 replicas each (row r of [0, 64 KiB): first halves at
//    [0, 128), second at [128, 256); a lane reads replica lane % 8), the V entry in bf16 (16 bytes) in 16
//    replicas (row r of [64 KiB, 128 KiB); replica lane % 16), so the 8 lanes of each quarter-warp
//    wavefront hit distinct banks and the keys need no bf16 unpacking (measured 3% faster).
//  * A warp takes a contiguous run of 16-token tiles.  Lane (g, t) = (lane / 4, lane % 4) owns tokens
//    t, t + 4, t + 8, t + 12 of each tile and pair-group g: channel group g (8 low channels) and its RoPE
//    partner group g + 8.  Its positions advance by 4 from token to token and from tile to tile, and
//    the rotation e^{i n w} of its 8 pairs follows the step-4 recurrence in difference form
//    (D_{j+1} = D_j - 4 sin^2(2w) X_j, X_{j+1} = X_j + D_{j+1}), set from the table every 32 tiles.
//  * Scores: the lane keeps the 4 query heads in the order h ^ hl, hl = 2 (g & 1) + ((g >> 1) & 1), so the
//    reduce-scatter over the 8 lanes of its t sends fixed registers: after exchanges over lane bits 2
//    and 3 the lane holds head hl of its 4 tokens, after bit 4 tokens 2 b, 2 b + 1 (b = g >> 2).
//  * Softmax: one lazy maximum per head, the same value in every lane that finishes that head.
//  * Values: out^T += Vhat^T P^T with mma.sync m16n8k16 (bf16 in, fp32 accumulate).  A fragments are the
//    gathered value entries re-paired across two tokens by byte permutes; the B fragment's 8 columns are
//    the 4 heads' weights split into bf16 hi and lo parts (column 2h + r).  Lane (g, t) accumulates head
//    t: rows g and g + 8 of every m-tile, hi and lo columns, all four registers in use.
//  * Index words arrive through a per-warp ring of 512-byte stages filled with 16-byte cp.async copies
//    (lane L copies chunk L of the tile) and are read with conflict-free 4-byte loads.
#pragma once

#include "decode_kernel.cuh"

namespace loopvq {

template <int WARPS, int DEPTH>
struct GqaSmem {
    static constexpr int QPK = 4;
    static constexpr uint32_t kTables = 131072u;
    static constexpr uint32_t kRing = kTables;
    static constexpr uint32_t kRingBytes = (uint32_t)WARPS * DEPTH * 512u;
    static constexpr uint32_t kRec = kRing + kRingBytes;
    static constexpr uint32_t kRecFloats = 128 + 4;                  // per (warp, head)
    static constexpr uint32_t kBytes = kRec + (uint32_t)WARPS * QPK * kRecFloats * 4u;
};

__device__ __forceinline__ float2 f2lo(const float4 &v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 f2hi(const float4 &v) { return make_float2(v.z, v.w); }

template <int WARPS, int MINB, int DEPTH>
__global__ void __launch_bounds__(WARPS * 32, MINB) decode_gqa_kernel(const DecodeArgs a) {
    constexpr int D = 128, NP = 8, QPK = 4;                // pair-groups = index words per token
    constexpr int NT = WARPS * 32;
    constexpr int ANCHOR = 32;                             // tiles between two settings from the table
    using S = GqaSmem<WARPS, DEPTH>;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ long long range_info[4];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    asm volatile("griddepcontrol.launch_dependents;");
    if (warp == 0) cta_range(a, lane, range_info);
    __syncthreads();
    long long pos = range_info[0];
    const long long x_end = range_info[1];
    long long seg0 = range_info[2];
    int h = (int)(range_info[3] >> 32), b = (int)(range_info[3] & 0xffffffffLL);

    const int g = lane >> 2, t = lane & 3;
    const int hl = 2 * (g & 1) + ((g >> 1) & 1);          // the head whose scores this lane finishes
    const int kb = g >> 2;                                 // ... for its tokens 2 kb, 2 kb + 1
    const uint32_t colk = (uint32_t)((lane & 7) * 16);     // the lane's K replica (first half; + 128 second)
    const uint32_t colv = 0x10000u | (uint32_t)((lane & 15) * 16);   // the lane's V replica (V table at 64 KiB)
    const uint32_t smem_base = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t ring = smem_base + S::kRing + (uint32_t)warp * DEPTH * 512u;
    float *rec = reinterpret_cast<float *>(smem + S::kRec) + warp * QPK * S::kRecFloats;
    // lanes finishing head h for tokens 0, 1 of this t (+ 16 for tokens 2, 3)
    const int hw = g >> 1;                                 // the head of this lane's B-fragment column
    const int src_b = 4 * ((hw >> 1) | ((hw & 1) << 1)) + t;
    const int src_c = 4 * ((t >> 1) | ((t & 1) << 1));     // a lane finishing head t (accumulator rescale)

    // recurrence coefficients of the lane's 8 pairs f = 8g + e: -4 sin^2 2w (table row 2)
    float2 nl[4];
    {
        const float4 s2a = __ldg(reinterpret_cast<const float4 *>(a.rope + 2 * D + D / 2 + 8 * g));
        const float4 s2b = __ldg(reinterpret_cast<const float4 *>(a.rope + 2 * D + D / 2 + 8 * g + 4));
        nl[0] = f2(-4.f * s2a.x * s2a.x, -4.f * s2a.y * s2a.y);
        nl[1] = f2(-4.f * s2a.z * s2a.z, -4.f * s2a.w * s2a.w);
        nl[2] = f2(-4.f * s2b.x * s2b.x, -4.f * s2b.y * s2b.y);
        nl[3] = f2(-4.f * s2b.z * s2b.z, -4.f * s2b.w * s2b.w);
    }

    int staged_h = -1;                                     // the KV head whose slices the tables hold
    while (pos < x_end && h < a.Hkv) {
        int len, st, base;
        const long long seg_end = seg0 + seq_tiles(a, b, base, st, len);
        const long long pend = seg_end < x_end ? seg_end : x_end;
        if (pend > pos) {
            const int piece = h * a.B + b + (int)blockIdx.x;
            const int tok_begin = base + 4 * (int)(pos - seg0);
            const int tok_end = min(base + 4 * (int)(pend - seg0), len);
            const int n4 = (int)(pend - pos);              // four-token tiles of the piece
            const int n16 = (n4 + 3) >> 2;
            __syncthreads();                               // the previous piece's tables and records are done

            // stage the slices of head h: K entry r in fp32 (32 bytes) at row r of [0, 64 KiB), its first
            // half in 8 replicas at bytes [0, 128), its second half in 8 replicas at [128, 256); V entry r
            // in bf16 (16 bytes) in 16 replicas at row r of [64 KiB, 128 KiB).  The slices depend on the KV
            // head only, so a piece of the head already staged keeps them.  Thread r reads entry r once and
            // writes its replicas starting at replica r mod 8 (16), so the 8 lanes of each quarter-warp
            // store write distinct banks.
            const bool restage = h != staged_h;
            if (restage) {
                const uint4 *sk = reinterpret_cast<const uint4 *>(a.slk + (size_t)h * a.K * 8);
                const uint4 *sv = reinterpret_cast<const uint4 *>(a.slv + (size_t)h * a.K * 8);
                for (int r = tid; r < 256; r += NT) {
                    uint4 ek = make_uint4(0u, 0u, 0u, 0u), ev = make_uint4(0u, 0u, 0u, 0u);
                    if (r < a.K) {
                        ek = __ldg(sk + r);
                        ev = __ldg(sv + r);
                    }
                    const float4 k0 = make_float4(bf16lo(ek.x), bf16hi(ek.x), bf16lo(ek.y), bf16hi(ek.y));
                    const float4 k1 = make_float4(bf16lo(ek.z), bf16hi(ek.z), bf16lo(ek.w), bf16hi(ek.w));
                    unsigned char *row = smem + r * 256;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        *reinterpret_cast<float4 *>(row + ((k + r) & 7) * 16) = k0;
                        *reinterpret_cast<float4 *>(row + 128 + ((k + r) & 7) * 16) = k1;
                    }
#pragma unroll
                    for (int k = 0; k < 16; ++k) *reinterpret_cast<uint4 *>(row + 65536 + ((k + r) & 15) * 16) = ev;
                }
                staged_h = h;
            }

            // the query heads in slot order s -> head s ^ hl, scaled, at the lane's channels
            float2 ql[QPK][4], qh[QPK][4];
#pragma unroll
            for (int s = 0; s < QPK; ++s) {
                const uint16_t *qp = a.q + ((size_t)b * a.Hq + h * QPK + (s ^ hl)) * D + 8 * g;
                const uint4 lo = __ldg(reinterpret_cast<const uint4 *>(qp));
                const uint4 hi = __ldg(reinterpret_cast<const uint4 *>(qp + D / 2));
                const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w}, hw4[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    ql[s][i] = f2(bf16lo(lw[i]) * a.qscale, bf16hi(lw[i]) * a.qscale);
                    qh[s][i] = f2(bf16lo(hw4[i]) * a.qscale, bf16hi(hw4[i]) * a.qscale);
                }
            }

            // this warp's run of 16-token tiles [i0, i1) of the piece
            const int i0 = (int)((long long)warp * n16 / WARPS), i1 = (int)((long long)(warp + 1) * n16 / WARPS);
            // index copies: lane L takes chunk L (four-tile L / 8, pair-group L % 8)
            const int kc = lane >> 3;
            const uint32_t *idx_b = a.idx + ((size_t)b * a.Hkv + h) * (size_t)a.Nmax * NP;
            const char *src = reinterpret_cast<const char *>(idx_b + ((size_t)((tok_begin >> 2) + 4 * i0 + kc) * NP + (lane & 7)) * 4);
            const uint32_t dst = ring + (uint32_t)lane * 16u;
            int crem = n4 - 4 * i0, ctl = i1 - i0;         // four-tiles of the piece / tiles of the warp, from the copy on
            auto copy_tile = [&](uint32_t soff) {
                const bool f0 = ctl > 0 && crem > kc;
                // a chunk outside the piece reads nothing (source size 0) from a valid address
                cp_async16_zfill(dst + soff, f0 ? src : reinterpret_cast<const char *>(a.idx), f0);
                cp_async_commit();
                src += 512;
                crem -= 4;
                --ctl;
            };
#pragma unroll
            for (int d = 0; d < DEPTH; ++d) copy_tile((uint32_t)d * 512u);

            float4 acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            float m = -1e30f, l = 0.f;                     // head hl: lazy maximum, sum of this lane's weights
            float2 xc[4], xs[4], dc[4], ds[4];             // e^{i n w} of the 8 pairs and its difference
            // the lane's finished tokens n = base_n + 2 kb + {0, 1} * 4 are attended iff 0 <= n - st < tok_end - st
            int nrel = tok_begin + 16 * i0 + t + 8 * kb - st;
            const unsigned span = (unsigned)(tok_end - st);
            const unsigned char *wrd = smem + S::kRing + (uint32_t)warp * DEPTH * 512u + 4u * (4 * g + t);
            uint32_t soff = 0;
            if (restage) __syncthreads();                  // tables staged (the condition is CTA-uniform)

            for (int ib = i0; ib < i1; ib += ANCHOR) {
                {
                    // X = e^{i n0 w} at the lane's first position, D = X (1 - e^{-4iw}) = X (2 sin^2 2w + i sin 4w)
                    const int n0 = tok_begin + 16 * ib + t;
                    const float *row = a.rope + (size_t)min(n0, a.Nmax - 1) * D + 8 * g;
                    const float4 c0 = __ldg(reinterpret_cast<const float4 *>(row));
                    const float4 c1 = __ldg(reinterpret_cast<const float4 *>(row + 4));
                    const float4 s0 = __ldg(reinterpret_cast<const float4 *>(row + D / 2));
                    const float4 s1 = __ldg(reinterpret_cast<const float4 *>(row + D / 2 + 4));
                    const float *r2 = a.rope + 2 * D + D / 2 + 8 * g, *r4 = a.rope + 4 * D + D / 2 + 8 * g;
                    const float4 a0 = __ldg(reinterpret_cast<const float4 *>(r2));
                    const float4 a1 = __ldg(reinterpret_cast<const float4 *>(r2 + 4));
                    const float4 b0 = __ldg(reinterpret_cast<const float4 *>(r4));
                    const float4 b1 = __ldg(reinterpret_cast<const float4 *>(r4 + 4));
                    const float2 cc[4] = {f2lo(c0), f2hi(c0), f2lo(c1), f2hi(c1)};
                    const float2 ss[4] = {f2lo(s0), f2hi(s0), f2lo(s1), f2hi(s1)};
                    const float2 s2[4] = {f2lo(a0), f2hi(a0), f2lo(a1), f2hi(a1)};
                    const float2 s4[4] = {f2lo(b0), f2hi(b0), f2lo(b1), f2hi(b1)};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 al = f2(2.f * s2[i].x * s2[i].x, 2.f * s2[i].y * s2[i].y);
                        xc[i] = cc[i];
                        xs[i] = ss[i];
                        // (c + i s)(al + i s4) = (c al - s s4) + i (c s4 + s al)
                        dc[i] = __ffma2_rn(cc[i], al, neg2(__fmul2_rn(ss[i], s4[i])));
                        ds[i] = __ffma2_rn(cc[i], s4[i], __fmul2_rn(ss[i], al));
                    }
                }

                const int ie = min(ib + ANCHOR, i1);
                for (int i = ib; i < ie; ++i) {
                    cp_async_wait<DEPTH - 1>();
                    __syncwarp();
                    const uint32_t *wp = reinterpret_cast<const uint32_t *>(wrd + soff);
                    uint32_t w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) w[k] = wp[32 * k];     // four-tile k, pair-group g, token t

                    // ---- keys: gather, rebuild, rotate once, score against the 4 heads
                    float sc[4][QPK];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t al = __byte_perm(w[k], colk, 0x7604), ah = __byte_perm(w[k], colk, 0x7614);
                        const float4 l0 = *reinterpret_cast<const float4 *>(smem + al);          // group g
                        const float4 l1 = *reinterpret_cast<const float4 *>(smem + al + 128);
                        const float4 h0 = *reinterpret_cast<const float4 *>(smem + ah);          // group g + 8
                        const float4 h1 = *reinterpret_cast<const float4 *>(smem + ah + 128);
                        const float2 klv[4] = {f2lo(l0), f2hi(l0), f2lo(l1), f2hi(l1)};
                        const float2 khv[4] = {f2lo(h0), f2hi(h0), f2lo(h1), f2hi(h1)};
                        float2 rl[4], rh[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 kl = klv[i], kh = khv[i];
                            rl[i] = __ffma2_rn(kl, xc[i], neg2(__fmul2_rn(kh, xs[i])));     // k_f cos - k_{f+D/2} sin
                            rh[i] = __ffma2_rn(kh, xc[i], __fmul2_rn(kl, xs[i]));           // k_{f+D/2} cos + k_f sin
                        }
#pragma unroll
                        for (int s = 0; s < QPK; ++s) {
                            float2 acc2 = __fmul2_rn(ql[s][0], rl[0]);
                            acc2 = __ffma2_rn(qh[s][0], rh[0], acc2);
#pragma unroll
                            for (int i = 1; i < 4; ++i) {
                                acc2 = __ffma2_rn(ql[s][i], rl[i], acc2);
                                acc2 = __ffma2_rn(qh[s][i], rh[i], acc2);
                            }
                            sc[k][s] = acc2.x + acc2.y;
                        }
                        // advance every pair by 4 positions
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            dc[i] = __ffma2_rn(nl[i], xc[i], dc[i]);
                            ds[i] = __ffma2_rn(nl[i], xs[i], ds[i]);
                            xc[i] = __fadd2_rn(xc[i], dc[i]);
                            xs[i] = __fadd2_rn(xs[i], ds[i]);
                        }
                    }
                    // the stage's words are in registers: refill it with the tile DEPTH ahead
                    __syncwarp();
                    copy_tile(soff);
                    soff = soff + 512u == DEPTH * 512u ? 0u : soff + 512u;

                    // ---- reduce-scatter over the 8 lanes of this t: slots 2, 3 go to the lane across bit 2,
                    // slot 1 across bit 3 (fixed registers); then tokens across bit 4
                    float e2[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float a0 = sc[k][0] + __shfl_xor_sync(0xffffffffu, sc[k][2], 4);
                        const float a1 = sc[k][1] + __shfl_xor_sync(0xffffffffu, sc[k][3], 4);
                        e2[k] = a0 + __shfl_xor_sync(0xffffffffu, a1, 8);
                    }
                    float sa, sb;                          // head hl, tokens 2 kb and 2 kb + 1
                    {
                        const float k0 = kb ? e2[2] : e2[0], k1 = kb ? e2[3] : e2[1];
                        const float o0 = kb ? e2[0] : e2[2], o1 = kb ? e2[1] : e2[3];
                        sa = k0 + __shfl_xor_sync(0xffffffffu, o0, 16);
                        sb = k1 + __shfl_xor_sync(0xffffffffu, o1, 16);
                    }
                    sa = (unsigned)nrel < span ? sa : -CUDART_INF_F;
                    sb = (unsigned)(nrel + 4) < span ? sb : -CUDART_INF_F;
                    nrel += 16;

                    // ---- online softmax, one lazy maximum per head
                    if (__any_sync(0xffffffffu, fmaxf(sa, sb) > m + 8.f)) {
                        float tmax = fmaxf(fmaxf(sa, sb), m);
                        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
                        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
                        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
                        const float corr = ex2(m - tmax);          // head hl
                        l *= corr;
                        m = tmax;
                        const float ct = __shfl_sync(0xffffffffu, corr, src_c);   // head t: this lane's accumulators
                        const float2 c2 = f2(ct, ct);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float2 lo2 = __fmul2_rn(f2(acc[j].x, acc[j].y), c2), hi2 = __fmul2_rn(f2(acc[j].z, acc[j].w), c2);
                            acc[j] = make_float4(lo2.x, lo2.y, hi2.x, hi2.y);
                        }
                    }
                    const float pa = ex2(sa - m), pb = ex2(sb - m);
                    l += pa + pb;

                    // ---- weights to the B fragment: column 2 h + r holds part r (0 hi, 1 lo) of head h
                    uint32_t bq0, bq1;
                    {
                        const float ha = __uint_as_float(__float_as_uint(pa) & 0xffff0000u);
                        const float hb = __uint_as_float(__float_as_uint(pb) & 0xffff0000u);
                        const uint32_t xa = cvt_bf16x2(pa - ha, ha), xb = cvt_bf16x2(pb - hb, hb);
                        const uint32_t yh = __byte_perm(xa, xb, 0x5410), yl = __byte_perm(xa, xb, 0x7632);
                        const uint32_t h0 = __shfl_sync(0xffffffffu, yh, src_b), l0 = __shfl_sync(0xffffffffu, yl, src_b);
                        const uint32_t h1 = __shfl_sync(0xffffffffu, yh, src_b + 16), l1 = __shfl_sync(0xffffffffu, yl, src_b + 16);
                        bq0 = (g & 1) ? l0 : h0;           // k-slots 2t, 2t + 1: tokens 0, 1 of this t
                        bq1 = (g & 1) ? l1 : h1;           // k-slots 2t + 8, 2t + 9: tokens 2, 3
                    }

                    // ---- values: m-tile j < 4 takes channels 2j, 2j + 1 of group g, j >= 4 those of group g + 8
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        uint4 v[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            v[k] = *reinterpret_cast<const uint4 *>(smem + __byte_perm(w[k], colv, u ? 0x7634u : 0x7624u));
                        const uint32_t v0[4] = {v[0].x, v[0].y, v[0].z, v[0].w}, v1[4] = {v[1].x, v[1].y, v[1].z, v[1].w};
                        const uint32_t v2[4] = {v[2].x, v[2].y, v[2].z, v[2].w}, v3[4] = {v[3].x, v[3].y, v[3].z, v[3].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16_16816(acc[4 * u + j], __byte_perm(v0[j], v1[j], 0x5410), __byte_perm(v0[j], v1[j], 0x7632),
                                           __byte_perm(v2[j], v3[j], 0x5410), __byte_perm(v2[j], v3[j], 0x7632), bq0, bq1);
                    }
                }
            }
            cp_async_wait<0>();

            // ---- the warp's records: lane (g, t) holds head t at rows g, g + 8 of every m-tile
            {
                float lsum = l;                            // head hl over the 8 lanes finishing it
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
                float *rt = rec + t * S::kRecFloats;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int ch = 8 * (g + 8 * (j >> 2)) + 2 * (j & 3);
                    rt[ch] = acc[j].x + acc[j].y;
                    rt[ch + 1] = acc[j].z + acc[j].w;
                }
                if (t == 0 && kb == 0) {                   // lanes 0, 4, 8, 12: heads hl = 0, 2, 1, 3
                    float *rh = rec + hl * S::kRecFloats;
                    rh[D] = lsum > 0.f ? m : -CUDART_INF_F;
                    rh[D + 1] = lsum;
                }
            }
            __syncthreads();
            // ---- combine the warps, write the piece's partial records
            {
                const float *recs = reinterpret_cast<const float *>(smem + S::kRec);
                for (int it = tid; it < QPK * D; it += NT) {
                    const int d = it % D, j = it / D;
                    float mx = -CUDART_INF_F;
                    for (int w2 = 0; w2 < WARPS; ++w2) mx = fmaxf(mx, recs[(w2 * QPK + j) * S::kRecFloats + D]);
                    float o = 0.f, lsum = 0.f;
                    if (mx != -CUDART_INF_F) {
                        for (int w2 = 0; w2 < WARPS; ++w2) {
                            const float *r = recs + (w2 * QPK + j) * S::kRecFloats;
                            const float wgt = ex2(r[D] - mx);
                            o += r[d] * wgt;
                            lsum += r[D + 1] * wgt;
                        }
                    }
                    const size_t rr = (size_t)piece * QPK + j;
                    a.ws_o[rr * D + d] = o;
                    if (d == 0) a.ws_ml[rr] = f2(mx, lsum);
                }
            }
            pos = pend;
        }
        seg0 = seg_end;
        if (++b == a.B) {
            b = 0;
            ++h;
        }
    }
}

}  // namespace loopvq
