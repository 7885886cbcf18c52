// Split-K decode attention over the loop-axis coded cache, one query head per KV head, D = 128,
// channel groups of 4 (the looped-decoder workloads): a kernel with 8 RoPE pairs per lane and the
// value accumulation on the tensor cores.
//
// LoopVQ paper, Sec. 4.3 "Attention" and App. C: every index is looked up in the loop step's
// codebook slice held in shared memory, keys are rebuilt before RoPE and rotated at their positions,
// and the tokens are cut into splits whose partial outputs are merged through their log-sum-exp.
//
// Design (B200, sm_100a):
//  * The tile space, pieces and partial records are those of decode_split_kernel (decode_kernel.cuh),
//    and the merge kernel (decode_merge.cuh) combines the records.  The slices are staged as bank-private replicas: row r
//    holds K entry r as 8 bytes of bf16 in 16 replicas and V entry r likewise (a lane reads replica
//    lane % 16, so the 16 lanes of a half-warp wavefront hit distinct banks).  Each gathered key entry is
//    widened to fp32 by one m16n8k8 tensor-core product with the identity (lane-local, exact), so the
//    key side needs no ALU unpacking and gathers 256 bytes per token and KV head instead of the 512 of
//    fp32 tables (4% faster at ctx32k than fp32 tables, once the value side below was in place; 6%
//    slower before it; with TaSQ keys 9% faster together with the value layout below, slower alone).
//  * A warp takes a contiguous run of 16-token tiles of the piece.  Lane (g, t) = (lane / 4, lane % 4)
//    owns the tokens t, t + 4, t + 8, t + 12 of each tile and the two pair-groups g and g + 8: the
//    channel groups g, g + 8 (low channels) and g + 16, g + 24 (their RoPE partners), 8 RoPE pairs.
//    Its positions advance by 4 from token to token and from tile to tile.
//  * Keys: the query is rotated instead of the keys, Z_f(n) = (q_f + i q_{f+D/2}) e^{-i n w_f}, and the
//    score is the sum over pairs of Re(Z_f) k_f + Im(Z_f) k_{f+D/2}.  Along a lane's positions Z follows
//    X_{j+1} = 2 cos(4w) X_j - X_{j-1}.  For the 4 high-frequency pairs (|sin 4w| bounded away from 0)
//    that is one fused multiply-add per component and step.  For the 4 low-frequency pairs the same
//    recurrence is run in the difference form D_{j+1} = D_j - 4 sin^2(2w) X_j, X_{j+1} = X_j + D_{j+1}
//    (Reinsch), whose coefficient keeps full relative precision as w -> 0.  Both are set from the
//    table every 64 tiles, which bounds the rounding drift to 256 steps (every 32 measured 1% slower).
//  * The lane's 4 partial scores are reduce-scattered over the 8 lanes of its t (3 exchanges); each
//    lane finishes one token.  The softmax maximum is one value per warp, lazy (it moves, with an exact
//    rescale, only when a score exceeds it by more than 8 in log2 units).
//  * Values on the tensor cores with mma.sync m16n8k16 (bf16 in, fp32 accumulate), 8 per 16-token tile:
//    one per (token octet, group octet u).  The k dimension is (token slot, channel parity) over slots t
//    and t + 4 of the octet, the A rows g and g + 8 are channels 0-1 and 2-3 of group 8u + g, so a lane's
//    A quad is exactly its two gathered 8-byte value entries (tokens t and t + 4, as loaded: no moves or
//    permutes).  B column g < 4 holds, at channel parity g & 1, the token's weight split into a bf16 hi
//    part (g < 2) or lo part, which represents the fp32 weight to about 2^-16 relative; columns 4-7 are
//    zero.  Lanes t = 0 and 1 accumulate the hi and lo parts of the same channels, added at the end.
//    (The first version put the weights in A with one token per MMA: 16 MMAs per tile with half the A
//    rows zero, whose A quads had to be assembled from separate registers; 7% slower at ctx32k.)
//  * Index words arrive through a per-warp ring of 1 KiB stages in shared memory filled with 16-byte
//    cp.async copies (lane L copies chunks L and L + 32 of the tile); each lane reads its 8 words with
//    conflict-free 4-byte loads.
//  * Groups of 16 channels (C = 16: the per-loop-step coding the LoopVQ paper compares against, Sec. 5.1,
//    "CQ") keep every lane's work: pair-group g's channels are quarter g % 4 of code group 4g / 16, its
//    RoPE partners the same quarter of group 4g / 16 + NP, and pair-group g + 8 is two groups on, so a
//    lane reads words g / 4 and g / 4 + 2 instead of g and g + 8 and gathers its 8 bytes at quarter g % 4
//    of the 32-byte entry.  Entries are staged in 4 replicas (replica t), rows stay 256 bytes, and the
//    ring stage is NP = 4 words per token (256 bytes per 16-token tile).
//  * TaSQ keys (TQ, LoopVQ paper App. B): word p's key codes are TaSQ groups 2p and 2p + 1, whose
//    entries hold the RoPE pairs of the head's pair order interleaved.  The lane's 8 pairs come from
//    that order, so all of them run the difference form; their rotated query is divided by the channel
//    weight, and the finished score is multiplied by the token's scale, read one tile ahead.
#pragma once

#include "decode_kernel.cuh"

namespace loopvq {

// Four bf16 channels (two packed words) widened to fp32 on the tensor core: an m16n8k8 product with the
// identity as B returns each lane's own A elements, so lane (g, t) gets (a0.lo, a0.hi, a1.lo, a1.hi).
// `eye` is the lane's identity fragment, B[2t][g] and B[2t + 1][g].
__device__ __forceinline__ float4 widen_bf16x4(uint2 e, uint32_t eye) {
    float4 c;
    asm("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, {%7, %7, %7, %7};"
        : "=f"(c.x), "=f"(c.y), "=f"(c.z), "=f"(c.w)
        : "r"(e.x), "r"(e.y), "r"(eye), "f"(0.f));
    return c;
}

// Shared memory of the kernel: K/V replicas, then the index ring (stages of SB bytes), then the warp
// records.
template <int WARPS, int DEPTH, uint32_t SB>
struct MhaSmem {
    static constexpr uint32_t kTables = 65536u;
    static constexpr uint32_t kRing = kTables;
    static constexpr uint32_t kRingBytes = (uint32_t)WARPS * DEPTH * SB;
    static constexpr uint32_t kRec = kRing + kRingBytes;
    static constexpr uint32_t kRecFloats = 128 + 4;
    static constexpr uint32_t kBytes = kRec + (uint32_t)WARPS * kRecFloats * 4u;
};

// TQ: keys coded after the TaSQ transform (LoopVQ paper, App. B).  Word p's key codes are TaSQ groups 2p
// and 2p + 1, whose entries hold complete RoPE pairs (f, f + D/2) of the low channels perm[4p .. 4p + 3]
// interleaved; the lane keeps one rotated query pair (re, im) per pair, divided by the channel weight,
// runs the difference-form recurrence on every pair, and multiplies each finished score by its token's
// scale sigma.
template <int WARPS, int MINB, int DEPTH, bool TQ = false, int C = 4>
__global__ void __launch_bounds__(WARPS * 32, MINB) decode_mha_kernel(const DecodeArgs a) {
    static_assert(C == 4 || (C == 16 && !TQ), "groups of 4 channels, or of 16 with plain keys");
    constexpr int D = 128, NP = D / (2 * C);               // index words per token
    constexpr uint32_t SB = 64u * NP;                      // bytes of one 16-token ring stage
    constexpr int NT = WARPS * 32;
    constexpr int ANCHOR = 64;                             // tiles between two settings from the table
    using S = MhaSmem<WARPS, DEPTH, SB>;

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
    // the lane's K column: C = 4, replica lane % 16 of the 8-byte entry; C = 16, quarter g % 4 of the
    // 32-byte entry in replica t (the 16 lanes of a half-warp read 16 distinct 8-byte slots of a row)
    const uint32_t colk = C == 4 ? (uint32_t)((lane & 15) * 8) : (uint32_t)(t * 32 + (g & 3) * 8);
    const uint32_t eye = ((2 * (lane & 3) == (lane >> 2)) ? 0x3F80u : 0u) |
                         ((2 * (lane & 3) + 1 == (lane >> 2)) ? 0x3F800000u : 0u);
    const uint32_t colv = colk + 128u;                     // and its V column
    const uint32_t smem_base = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t ring = smem_base + S::kRing + (uint32_t)warp * DEPTH * SB;
    float *rec = reinterpret_cast<float *>(smem + S::kRec) + warp * S::kRecFloats;

    // recurrence coefficients of the lane's pairs: high pairs f = 4g + e (2 cos 4w), low pairs
    // f = 32 + 4g + e (-4 sin^2 2w); from table rows 4 and 2
    float2 tcA[2], nlB[2];
    {
        const float4 c4 = __ldg(reinterpret_cast<const float4 *>(a.rope + 4 * D + 4 * g));
        const float4 s2 = __ldg(reinterpret_cast<const float4 *>(a.rope + 2 * D + D / 2 + 32 + 4 * g));
        tcA[0] = f2(2.f * c4.x, 2.f * c4.y);
        tcA[1] = f2(2.f * c4.z, 2.f * c4.w);
        nlB[0] = f2(-4.f * s2.x * s2.x, -4.f * s2.y * s2.y);
        nlB[1] = f2(-4.f * s2.z * s2.z, -4.f * s2.w * s2.w);
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

            // stage: row r = K entry r in bf16, 16 replicas of 8 bytes at [0, 128); V entry r likewise at
            // [128, 256).  The slices depend on the KV head only, so a piece of the head already staged (the
            // next sequence of the same head) keeps them.  Thread r reads entry r once and writes its
            // replicas starting at replica r mod 16, so the lanes of each half-warp store write distinct
            // banks.
            const bool restage = h != staged_h;
            if (restage) {
                const uint16_t *sk = a.slk + (size_t)h * a.K * C;
                const uint16_t *sv = a.slv + (size_t)h * a.K * C;
                for (int r = tid; r < 256; r += NT) {
                    unsigned char *row = smem + r * 256;
                    if constexpr (C == 4) {
                        uint2 ek = make_uint2(0u, 0u), ev = make_uint2(0u, 0u);
                        if (r < a.K) {
                            ek = __ldg(reinterpret_cast<const uint2 *>(sk + (size_t)r * 4));
                            ev = __ldg(reinterpret_cast<const uint2 *>(sv + (size_t)r * 4));
                        }
#pragma unroll
                        for (int k = 0; k < 16; ++k) *reinterpret_cast<uint2 *>(row + ((k + r) & 15) * 8) = ek;
#pragma unroll
                        for (int k = 0; k < 16; ++k) *reinterpret_cast<uint2 *>(row + 128 + ((k + r) & 15) * 8) = ev;
                    } else {
                        // 32-byte entries, 4 replicas each in [0, 128) (K) and [128, 256) (V)
                        uint4 e[4] = {};
                        if (r < a.K) {
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                e[j] = __ldg(reinterpret_cast<const uint4 *>(sk + (size_t)r * 16) + j);
                                e[2 + j] = __ldg(reinterpret_cast<const uint4 *>(sv + (size_t)r * 16) + j);
                            }
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t o = (uint32_t)((k + r) & 3) * 32u;
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                *reinterpret_cast<uint4 *>(row + o + 16 * j) = e[j];
                                *reinterpret_cast<uint4 *>(row + 128 + o + 16 * j) = e[2 + j];
                            }
                        }
                    }
                }
                staged_h = h;
            }

            // this warp's run of 16-token tiles [i0, i1) of the piece
            const int i0 = (int)((long long)warp * n16 / WARPS), i1 = (int)((long long)(warp + 1) * n16 / WARPS);
            const int kown = 2 * (g & 1) + ((g >> 1) & 1);  // the token (0..3) this lane finishes
            // Value products (below), selector of the packed weight x = {hi part: bytes 0-1, lo part: 2-3}:
            // B column g < 4 takes part g >> 1 in half g & 1, columns 4..7 are zero.
            const uint32_t sel0 =
                g >= 4 ? 0x4444u : ((g & 2) ? ((g & 1) ? 0x3244u : 0x4432u) : ((g & 1) ? 0x1044u : 0x4410u));
            // index copies: a stage is 4 NP chunks of 16 bytes (the 4 tokens of one four-tile and word),
            // in memory order; lane L takes chunk L (four-tile L / NP) and, with C = 4, chunk L + 32
            // (four-tile L / NP + 2).  With C = 16 the 16 chunks go to lanes 0..15.
            const int kc = lane / NP;
            const bool copier = C == 4 || lane < 16;
            const uint32_t *idx_b = a.idx + ((size_t)b * a.Hkv + h) * (size_t)a.Nmax * NP;
            const char *src = reinterpret_cast<const char *>(idx_b + (size_t)((tok_begin >> 2) + 4 * i0) * NP * 4) + lane * 16;
            const uint32_t dst = ring + (uint32_t)lane * 16u;
            int crem = n4 - 4 * i0, ctl = i1 - i0;         // four-tiles of the piece / tiles of the warp, from the copy on
            auto copy_tile = [&](uint32_t soff) {
                // a chunk outside the piece reads nothing (source size 0) from a valid address
                const bool f0 = ctl > 0 && crem > kc;
                if (copier) cp_async16_zfill(dst + soff, f0 ? src : reinterpret_cast<const char *>(a.idx), f0);
                if constexpr (C == 4) {
                    const bool f1 = ctl > 0 && crem > kc + 2;
                    cp_async16_zfill(dst + soff + 512u, f1 ? src + 512 : reinterpret_cast<const char *>(a.idx), f1);
                }
                cp_async_commit();
                src += SB;
                crem -= 4;
                --ctl;
            };
#pragma unroll
            for (int d = 0; d < DEPTH; ++d) copy_tile((uint32_t)d * SB);

            float4 acc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            float m = -1e30f, l = 0.f;
            float2 zar[2], zai[2], par[2], pai[2];         // high pairs: X_j and X_{j-1} (re, im)
            float2 zbr[2], zbi[2], dbr[2], dbi[2];         // low pairs: X_j and D_j = X_j - X_{j-1}
            float2 xq[8], dq[8], nq[8];                    // TQ: per pair (re, im) of X_j and D_j, -4 sin^2 2w
            if constexpr (TQ) {
                const int16_t *pm = a.tperm + (size_t)h * (D / 2);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int f = __ldg(pm + (j < 4 ? 4 * g + j : 32 + 4 * g + j - 4)) & (D / 2 - 1);
                    const float s2 = __ldg(a.rope + 2 * D + D / 2 + f);
                    nq[j] = f2(-4.f * s2 * s2, -4.f * s2 * s2);
                }
            }
            // the lane's finished token n is attended iff 0 <= n - st < tok_end - st
            int nrel = tok_begin + 16 * i0 + t + 4 * kown - st;
            const unsigned span = (unsigned)(tok_end - st);
            // TQ: the TaSQ scale of the token a lane finishes, loaded one tile ahead (0 outside the span,
            // where the score is masked anyway)
            const uint16_t *sig_b = TQ ? a.tsig + (size_t)b * a.Nmax + st : nullptr;
            auto load_sig = [&](int nr) {
                return (unsigned)nr < span ? __half2float(__ushort_as_half(__ldg(sig_b + nr))) : 0.f;
            };
            float sig_next = 0.f;
            if constexpr (TQ) sig_next = load_sig(nrel);
            // the lane's words: token t of pair-group g's word 4g / C and of pair-group g + 8's word
            const unsigned char *wrd = smem + S::kRing + (uint32_t)warp * DEPTH * SB + 4u * (4 * (4 * g / C) + t);
            uint32_t soff = 0;
            if (restage) __syncthreads();                  // tables staged (the condition is CTA-uniform)

            for (int ib = i0; ib < i1; ib += ANCHOR) {
                if constexpr (TQ) {
                    // X = (q_f + i q_{f+D/2}) / w_f e^{-i n0 w_f} at the lane's permuted pairs, D = X (2 sin^2 2w
                    // - i sin 4w)
                    const int n0 = tok_begin + 16 * ib + t;
                    const float *row = a.rope + (size_t)min(n0, a.Nmax - 1) * D;
                    const uint16_t *qp = a.q + ((size_t)b * a.Hq + h) * D;
                    const int16_t *pm = a.tperm + (size_t)h * (D / 2);
                    const float *wp = a.tw + (size_t)h * D;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int f = __ldg(pm + (j < 4 ? 4 * g + j : 32 + 4 * g + j - 4)) & (D / 2 - 1);
                        const float sc = a.qscale / __ldg(wp + f);
                        const float qf = bf16_to_f32(__ldg(qp + f)) * sc, qh = bf16_to_f32(__ldg(qp + D / 2 + f)) * sc;
                        const float c = __ldg(row + f), sn = __ldg(row + D / 2 + f);
                        const float s2 = __ldg(a.rope + 2 * D + D / 2 + f), s4 = __ldg(a.rope + 4 * D + D / 2 + f);
                        const float al = 2.f * s2 * s2;
                        const float zr = fmaf(qf, c, qh * sn), zi = fmaf(qh, c, -(qf * sn));
                        xq[j] = f2(zr, zi);
                        dq[j] = f2(fmaf(zr, al, zi * s4), fmaf(zi, al, -(zr * s4)));
                    }
                } else {
                    // X at the lane's first position n0 from the table and the query; the second state from
                    // X(n0 - 4) = X(n0) e^{+4iw}
                    const int n0 = tok_begin + 16 * ib + t;
                    const float *row = a.rope + (size_t)min(n0, a.Nmax - 1) * D;
                    const uint16_t *qp = a.q + ((size_t)b * a.Hq + h) * D;
                    const float4 cA = __ldg(reinterpret_cast<const float4 *>(row + 4 * g));
                    const float4 sA = __ldg(reinterpret_cast<const float4 *>(row + D / 2 + 4 * g));
                    const float4 cB = __ldg(reinterpret_cast<const float4 *>(row + 32 + 4 * g));
                    const float4 sB = __ldg(reinterpret_cast<const float4 *>(row + D / 2 + 32 + 4 * g));
                    const uint2 qal = __ldg(reinterpret_cast<const uint2 *>(qp + 4 * g));
                    const uint2 qah = __ldg(reinterpret_cast<const uint2 *>(qp + D / 2 + 4 * g));
                    const uint2 qbl = __ldg(reinterpret_cast<const uint2 *>(qp + 32 + 4 * g));
                    const uint2 qbh = __ldg(reinterpret_cast<const uint2 *>(qp + D / 2 + 32 + 4 * g));
                    const float4 c4A = __ldg(reinterpret_cast<const float4 *>(a.rope + 4 * D + 4 * g));
                    const float4 s4A = __ldg(reinterpret_cast<const float4 *>(a.rope + 4 * D + D / 2 + 4 * g));
                    const float4 s4B = __ldg(reinterpret_cast<const float4 *>(a.rope + 4 * D + D / 2 + 32 + 4 * g));
                    const float4 s2B = __ldg(reinterpret_cast<const float4 *>(a.rope + 2 * D + D / 2 + 32 + 4 * g));
                    const float qs = a.qscale;
                    const float2 ql[2][2] = {{f2(bf16lo(qal.x) * qs, bf16hi(qal.x) * qs), f2(bf16lo(qal.y) * qs, bf16hi(qal.y) * qs)},
                                             {f2(bf16lo(qbl.x) * qs, bf16hi(qbl.x) * qs), f2(bf16lo(qbl.y) * qs, bf16hi(qbl.y) * qs)}};
                    const float2 qh[2][2] = {{f2(bf16lo(qah.x) * qs, bf16hi(qah.x) * qs), f2(bf16lo(qah.y) * qs, bf16hi(qah.y) * qs)},
                                             {f2(bf16lo(qbh.x) * qs, bf16hi(qbh.x) * qs), f2(bf16lo(qbh.y) * qs, bf16hi(qbh.y) * qs)}};
                    const float2 cs[2][2] = {{f2(cA.x, cA.y), f2(cA.z, cA.w)}, {f2(cB.x, cB.y), f2(cB.z, cB.w)}};
                    const float2 sn[2][2] = {{f2(sA.x, sA.y), f2(sA.z, sA.w)}, {f2(sB.x, sB.y), f2(sB.z, sB.w)}};
                    float2 zr[2][2], zi[2][2];
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            // Z = (ql + i qh)(cos - i sin)
                            zr[u][e] = __ffma2_rn(ql[u][e], cs[u][e], __fmul2_rn(qh[u][e], sn[u][e]));
                            zi[u][e] = __ffma2_rn(qh[u][e], cs[u][e], __fmul2_rn(neg2(ql[u][e]), sn[u][e]));
                        }
                    const float2 c4[2] = {f2(c4A.x, c4A.y), f2(c4A.z, c4A.w)};
                    const float2 s4[2] = {f2(s4A.x, s4A.y), f2(s4A.z, s4A.w)};
                    const float2 sb4[2] = {f2(s4B.x, s4B.y), f2(s4B.z, s4B.w)};
                    const float2 al[2] = {f2(2.f * s2B.x * s2B.x, 2.f * s2B.y * s2B.y),
                                          f2(2.f * s2B.z * s2B.z, 2.f * s2B.w * s2B.w)};
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        zar[e] = zr[0][e];
                        zai[e] = zi[0][e];
                        // X(n0 - 4) = X (cos 4w + i sin 4w)
                        par[e] = __ffma2_rn(zr[0][e], c4[e], __fmul2_rn(neg2(zi[0][e]), s4[e]));
                        pai[e] = __ffma2_rn(zi[0][e], c4[e], __fmul2_rn(zr[0][e], s4[e]));
                        zbr[e] = zr[1][e];
                        zbi[e] = zi[1][e];
                        // D = X (1 - e^{4iw}) = X (2 sin^2 2w - i sin 4w)
                        dbr[e] = __ffma2_rn(zr[1][e], al[e], __fmul2_rn(zi[1][e], sb4[e]));
                        dbi[e] = __ffma2_rn(zi[1][e], al[e], __fmul2_rn(neg2(zr[1][e]), sb4[e]));
                    }
                }

                const int ie = min(ib + ANCHOR, i1);
                for (int i = ib; i < ie; ++i) {
                    cp_async_wait<DEPTH - 1>();
                    __syncwarp();
                    float sig = 0.f;
                    if constexpr (TQ) {
                        sig = sig_next;
                        sig_next = load_sig(nrel + 16);
                    }
                    const uint32_t *wp = reinterpret_cast<const uint32_t *>(wrd + soff);
                    uint32_t wa[4], wb[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        wa[k] = wp[4 * NP * k];            // four-tile k, pair-group g, token t
                        wb[k] = wp[4 * NP * k + 128 / C];  // pair-group g + 8: word 4g / C + 32 / C
                    }

                    // ---- keys: gather, rebuild, score the lane's 4 tokens over its 8 pairs
                    float s[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float4 e0 = widen_bf16x4(lds64(smem, __byte_perm(wa[k], colk, 0x7604)), eye);
                        const float4 e1 = widen_bf16x4(lds64(smem, __byte_perm(wa[k], colk, 0x7614)), eye);
                        const float4 e2 = widen_bf16x4(lds64(smem, __byte_perm(wb[k], colk, 0x7604)), eye);
                        const float4 e3 = widen_bf16x4(lds64(smem, __byte_perm(wb[k], colk, 0x7614)), eye);
                        if constexpr (TQ) {
                            // entries (u_f, u_{f+D/2}, u_f', u_{f'+D/2}): one packed FMA per pair
                            float2 sc2 = __fmul2_rn(xq[0], f2(e0.x, e0.y));
                            sc2 = __ffma2_rn(xq[1], f2(e0.z, e0.w), sc2);
                            sc2 = __ffma2_rn(xq[2], f2(e1.x, e1.y), sc2);
                            sc2 = __ffma2_rn(xq[3], f2(e1.z, e1.w), sc2);
                            sc2 = __ffma2_rn(xq[4], f2(e2.x, e2.y), sc2);
                            sc2 = __ffma2_rn(xq[5], f2(e2.z, e2.w), sc2);
                            sc2 = __ffma2_rn(xq[6], f2(e3.x, e3.y), sc2);
                            sc2 = __ffma2_rn(xq[7], f2(e3.z, e3.w), sc2);
                            s[k] = sc2.x + sc2.y;
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                dq[j] = __ffma2_rn(nq[j], xq[j], dq[j]);
                                xq[j] = __fadd2_rn(xq[j], dq[j]);
                            }
                            continue;
                        }
                        float2 sc2 = __fmul2_rn(zar[0], f2(e0.x, e0.y));
                        sc2 = __ffma2_rn(zar[1], f2(e0.z, e0.w), sc2);
                        sc2 = __ffma2_rn(zai[0], f2(e1.x, e1.y), sc2);
                        sc2 = __ffma2_rn(zai[1], f2(e1.z, e1.w), sc2);
                        sc2 = __ffma2_rn(zbr[0], f2(e2.x, e2.y), sc2);
                        sc2 = __ffma2_rn(zbr[1], f2(e2.z, e2.w), sc2);
                        sc2 = __ffma2_rn(zbi[0], f2(e3.x, e3.y), sc2);
                        sc2 = __ffma2_rn(zbi[1], f2(e3.z, e3.w), sc2);
                        s[k] = sc2.x + sc2.y;
                        // advance every pair by 4 positions
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float2 nr = __ffma2_rn(tcA[e], zar[e], neg2(par[e]));
                            const float2 ni = __ffma2_rn(tcA[e], zai[e], neg2(pai[e]));
                            par[e] = zar[e];
                            pai[e] = zai[e];
                            zar[e] = nr;
                            zai[e] = ni;
                            dbr[e] = __ffma2_rn(nlB[e], zbr[e], dbr[e]);
                            dbi[e] = __ffma2_rn(nlB[e], zbi[e], dbi[e]);
                            zbr[e] = __fadd2_rn(zbr[e], dbr[e]);
                            zbi[e] = __fadd2_rn(zbi[e], dbi[e]);
                        }
                    }
                    // the stage's words are in registers: refill it with the tile DEPTH ahead
                    __syncwarp();
                    copy_tile(soff);
                    soff = soff + SB == DEPTH * SB ? 0u : soff + SB;

                    // ---- reduce-scatter over the 8 lanes of this t: lane (g, t) ends with token kown
                    float sk;
                    {
                        const bool b1 = (g & 1) != 0, b2 = (g & 2) != 0;
                        const float k0 = b1 ? s[2] : s[0], k1 = b1 ? s[3] : s[1];
                        const float o0 = b1 ? s[0] : s[2], o1 = b1 ? s[1] : s[3];
                        const float a0 = k0 + __shfl_xor_sync(0xffffffffu, o0, 4);
                        const float a1 = k1 + __shfl_xor_sync(0xffffffffu, o1, 4);
                        const float kk = b2 ? a1 : a0, oo = b2 ? a0 : a1;
                        sk = kk + __shfl_xor_sync(0xffffffffu, oo, 8);
                        sk += __shfl_xor_sync(0xffffffffu, sk, 16);
                    }
                    if constexpr (TQ) sk *= sig;          // the finished token's TaSQ scale
                    sk = (unsigned)nrel < span ? sk : -CUDART_INF_F;
                    nrel += 16;

                    // ---- online softmax, one lazy maximum per warp
                    if (__any_sync(0xffffffffu, sk > m + 8.f)) {
                        float tmax = sk;
#pragma unroll
                        for (int o = 16; o >= 1; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
                        const float corr = ex2(m - tmax);
                        l *= corr;
                        const float2 c2 = f2(corr, corr);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 lo2 = __fmul2_rn(f2(acc[j].x, acc[j].y), c2);
                            acc[j].x = lo2.x;
                            acc[j].y = lo2.y;
                            const float2 hi2 = __fmul2_rn(f2(acc[j].z, acc[j].w), c2);
                            acc[j].z = hi2.x;
                            acc[j].w = hi2.y;
                        }
                        m = tmax;
                    }
                    const float p = ex2(sk - m);
                    l += p;

                    // ---- weights: token k's {bf16 hi, bf16 lo} (about 2^-16 of the fp32 weight together) from
                    // the lane 4 g'(k) + t that finished it
                    uint32_t xk[4];
                    {
                        const float hv = __uint_as_float(__float_as_uint(p) & 0xffff0000u);
                        const uint32_t x = cvt_bf16x2(p - hv, hv);        // upper: lo part, lower: hi part
                        xk[0] = __shfl_sync(0xffffffffu, x, t);
                        xk[1] = __shfl_sync(0xffffffffu, x, 8 + t);
                        xk[2] = __shfl_sync(0xffffffffu, x, 4 + t);
                        xk[3] = __shfl_sync(0xffffffffu, x, 12 + t);
                    }
                    // ---- values: A rows g, g + 8 = channels 0-1, 2-3 of group 8u + g; k = (token slot, channel
                    // parity) over slots t (k 2t, 2t + 1) and t + 4 (k 2t + 8, 2t + 9) of a token octet, so the
                    // lane's A quad is its two gathered 8-byte entries as loaded; B column g < 4 = (part g >> 1,
                    // parity g & 1) holds the slot's weight part at that parity
                    uint32_t bw[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) bw[k] = __byte_perm(xk[k], 0u, sel0);
#pragma unroll
                    for (int o = 0; o < 2; ++o) {
                        uint2 v[2][4];
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                v[j][u] = lds64(smem, __byte_perm((u & 1) ? wb[2 * o + j] : wa[2 * o + j], colv,
                                                                  (u < 2) ? 0x7624u : 0x7634u));
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            mma_bf16_16816(acc[u], v[0][u].x, v[0][u].y, v[1][u].x, v[1][u].y, bw[2 * o],
                                           bw[2 * o + 1]);
                    }
                }
            }
            cp_async_wait<0>();

            // ---- the warp's record
            {
                float lsum = l;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
                lsum *= 0.5f;                              // every token is finished by two lanes
                // lane (g, 0) holds the hi parts of channels 0-3 of group 8u + g, lane (g, 1) the lo parts
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float4 c = acc[u];
                    c.x += __shfl_xor_sync(0xffffffffu, c.x, 1);
                    c.y += __shfl_xor_sync(0xffffffffu, c.y, 1);
                    c.z += __shfl_xor_sync(0xffffffffu, c.z, 1);
                    c.w += __shfl_xor_sync(0xffffffffu, c.w, 1);
                    if (t == 0) *reinterpret_cast<float4 *>(rec + 4 * (8 * u + g)) = c;
                }
                if (lane == 0) {
                    rec[D] = lsum > 0.f ? m : -CUDART_INF_F;
                    rec[D + 1] = lsum;
                }
            }
            __syncthreads();
            // ---- combine the warps, write the piece's partial record
            {
                const float *recs = reinterpret_cast<const float *>(smem + S::kRec);
                for (int d = tid; d < D; d += NT) {
                    float mx = -CUDART_INF_F;
                    for (int w = 0; w < WARPS; ++w) mx = fmaxf(mx, recs[w * S::kRecFloats + D]);
                    float o = 0.f, lsum = 0.f;
                    if (mx != -CUDART_INF_F) {
                        for (int w = 0; w < WARPS; ++w) {
                            const float *r = recs + w * S::kRecFloats;
                            const float wgt = ex2(r[D] - mx);
                            o += r[d] * wgt;
                            lsum += r[D + 1] * wgt;
                        }
                    }
                    a.ws_o[(size_t)piece * D + d] = o;
                    if (d == 0) a.ws_ml[piece] = f2(mx, lsum);
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
