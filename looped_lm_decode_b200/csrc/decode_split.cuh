// Split-K decode attention over the loop-axis coded cache: the general kernel (every D, c, query-head
// ratio, codebook layout and key coding the library accepts).
//
// LoopVQ paper, Sec. 4.3 "Attention" and App. C: at loop step t every index is
// looked up in that step's codebook slice B_t held in shared memory, keys are
// rebuilt before RoPE and rotated from per-position cos/sin values, and the
// quantized tokens are cut into splits processed by separate thread blocks whose
// partial outputs are merged through their log-sum-exp (exact softmax).
//
// B200 design (not the pages' kernel):
//  * Exactly one wave of resident CTAs, sharing the 4-token tiles of all (KV head,
//    sequence) segments evenly whatever the sequence lengths (see the tile-space
//    helpers below): a CTA walks its tile range segment by segment, and each part
//    of a segment it covers (a piece) is one split of that segment, with its own
//    partial record for the log-sum-exp merge.
//  * For each piece the head's K and V slices are staged as bank-private replicas: row r (256 bytes) holds entry r of the K
//    slice in bytes [0,128) and of the V slice in [128,256), replicated so that
//    the 8-byte piece a lane reads sits in its own bank pair: lane l reads bytes
//    (l % 16) * 8 of the half-row.  For c = 4 that is replica l % 16 of the
//    8-byte entry; for c = 4j it is part l % j of replica (l % 16) / j of the
//    2c-byte entry (c = 8, 16, 32).  A gather by 16 lanes of random entries is conflict-free,
//    and its address is one byte permute of the index word (code -> bits 8..15,
//    the lane's column -> bits 0..7).
//  * Every lane owns 8 channels: 4 of a channel group g < D/(2c) and the 4
//    RoPE partners in group g + D/(2c), so all RoPE arithmetic stays in the
//    lane.  A token slot of D/8 lanes covers the head dimension and handles
//    4-token tiles; the 4 partial scores are reduce-scattered over the slot so
//    each lane finishes one token and takes one exponent.
//  * With one query head per KV head the query is rotated instead of the keys
//    (ROTQ): per pair f the score term is Re(Z) k_f + Im(Z) k_{f+D/2} with
//    Z = (q_f + i q_{f+D/2}) e^{-i p w_f}, and Z advances one position by one
//    complex multiply.  With several query heads the rebuilt keys are rotated
//    once and shared.
//  * Each thread keeps a DEPTH-deep queue of its own 16-byte index-word loads in
//    flight with cp.async (it reads back only what it copied, so no barrier is
//    involved).
//  * RoPE values: one table row per tile; the next position is one complex multiply away, and the
//    rest of the tile follows the three-term recurrence X_{k+1} = 2 cos(w) X_k - X_{k-1}, which holds
//    for every sequence X_k = A e^{-i k w} and needs one fused multiply-add per component.
//  * The tile's value gathers are issued before the key arithmetic, so their shared-memory latency
//    overlaps the score, reduction and softmax work.
//  * Online softmax with a lazy maximum; fp32 math in packed pairs (FFMA2).
#pragma once

#include "decode_kernel.cuh"

namespace loopvq {

// PG: one codebook per channel group.  The loop step's slice is then code-major with row r holding
// entry r of every group's codebook (D bf16), so each lane reads its own channels of the row and the
// 16 lanes of a token slot fall into distinct banks without replicas.  Tables: D = 128, K rows of 256 B
// at [0, 64 KiB) and V rows at [64 KiB, 128 KiB); D = 64, rows of 256 B holding K then V, in two
// copies whose second is rotated by 64 B within each half-row for the odd token slots of a half-warp.
// The table choice rides in the upper bytes of the gather column, which the byte permute passes on.
// TQ: keys coded with TaSQ (LoopVQ paper, App. B): the lane's two key codes are TaSQ groups 2p and
// 2p + 1, whose entries interleave complete RoPE pairs (f, f + D/2) of low channels taken from the
// permutation; the query is gathered at those channels and divided by the channel weights, the RoPE
// values come from those columns of the table, and each token's score is multiplied by its scale.
// XR: the RoPE values at each iteration's first token are carried from the previous iteration (one
// complex multiply by e^{-+i STRIDE w}) and set from the table every 16 iterations, instead of loading
// the table row one iteration ahead.
template <int D, int C, int QPK, int WARPS, int MINB, int DEPTH, int NW, bool PG = false, bool TQ = false,
          bool XR = false>
__global__ void __launch_bounds__(WARPS * 32, MINB) decode_split_kernel(const DecodeArgs a) {
    constexpr bool ROTQ = QPK == 1;                        // rotate the query, not every key
    constexpr int NP = D / (2 * C);                        // pair-groups = index words per token
    constexpr int HALVES = C / 4;                          // lanes sharing one pair-group
    constexpr int NL = D / 8;                              // lanes per token slot
    constexpr int SPW = 32 / NL;                           // slots per warp
    constexpr int NSLOT = WARPS * SPW;
    constexpr int NT = WARPS * 32;
    constexpr int EB = 2 * C;                              // bytes of one slice entry
    constexpr int REPL = 128 / EB;                         // replicas per half-row
    constexpr int TT = 4 * NW;                             // tokens per slot iteration
    constexpr int STRIDE = NSLOT * TT;                     // tokens between two iterations of a slot
    constexpr int QB = NT * 16 * NW;                       // bytes of one prefetch-queue stage
    constexpr uint32_t TBL = PG ? 131072u : 65536u;        // bytes of the staged K/V tables
    // With at most 2 query heads per KV head the slot records get their own shared memory after the
    // index queue, so a CTA keeps its tables across pieces of one KV head (its next piece is usually the
    // next sequence of the same head); otherwise they reuse the tables, which are staged every piece.
    constexpr bool KEEP = QPK <= 2;
    constexpr uint32_t REC_OFF = TBL + (uint32_t)DEPTH * QB;
    static_assert(C == 4 || C == 8 || C == 16 || C == 32, "c");
    static_assert(NL >= 8 && NL <= 16, "slot width");

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ long long range_info[4];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the merge kernel may be scheduled now; it waits for this grid before reading any record
    asm volatile("griddepcontrol.launch_dependents;");
    if (warp == 0) cta_range(a, lane, range_info);
    __syncthreads();
    long long pos = range_info[0];                         // next tile of this CTA
    const long long x_end = range_info[1];
    long long seg0 = range_info[2];                        // first tile of segment (h, b)
    int h = (int)(range_info[3] >> 32), b = (int)(range_info[3] & 0xffffffffLL);

    const int ls = lane % NL;                              // lane within the slot
    const int gp = ls / HALVES;                            // pair-group
    const int half = ls % HALVES;                          // which 4 channels of the group
    const int slot = warp * SPW + lane / NL;
    const unsigned slot_mask = ((1u << NL) - 1u) << (lane & ~(NL - 1));
    const int slot_lane0 = lane & ~(NL - 1);
    // gather columns of the K / V entries of the lane's group (lo) and of its RoPE partner group (hi)
    uint32_t colk_lo, colk_hi, colv_lo, colv_hi;
    if constexpr (!PG) {
        colk_lo = colk_hi = (uint32_t)((lane % 16) * 8);   // its own replica's 8-byte column
        colv_lo = colv_hi = colk_lo + 128u;
    } else if constexpr (D == 128) {
        const uint32_t cb = (uint32_t)((gp * C + half * 4) * 2);
        colk_lo = cb;
        colk_hi = cb + 128u;
        colv_lo = 0x10000u + cb;
        colv_hi = 0x10000u + cb + 128u;
    } else {
        const uint32_t odd = (uint32_t)((lane >> 3) & 1);  // second token slot of the half-warp
        const uint32_t cb = (uint32_t)((gp * C + half * 4) * 2);
        colk_lo = (odd << 16) | ((cb + 64u * odd) & 127u);
        colk_hi = (odd << 16) | ((cb + 64u + 64u * odd) & 127u);
        colv_lo = colk_lo + 128u;
        colv_hi = colk_hi + 128u;
    }
    const int ch = gp * C + half * 4;                      // first of this lane's 4 low channels

    int staged_h = -1;                                     // the KV head whose slices the tables hold
    // the pieces of this CTA, segment by segment
    while (pos < x_end && h < a.Hkv) {
        int len, st, base;
        const long long seg_end = seg0 + seq_tiles(a, b, base, st, len);
        const long long pend = seg_end < x_end ? seg_end : x_end;
        if (pend > pos) {
            const int piece = h * a.B + b + (int)blockIdx.x;
            // tokens [st, len) are attended; this piece covers the tiles [pos, pend) of the segment
            const int tok_begin = base + 4 * (int)(pos - seg0);
            const int tok_end = min(base + 4 * (int)(pend - seg0), len);
            __syncthreads();                               // the previous piece's slot records have been read

            // low channels of the lane's 4 RoPE pairs: ch .. ch+3, or under TaSQ the pairs 2*half, 2*half + 1
            // of TaSQ groups 2*gp (key code lo) and 2*gp + 1 (key code hi)
            int fq[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if constexpr (TQ) {
                    const int16_t *pm = a.tperm + (size_t)h * (D / 2);
                    fq[k] = __ldg(pm + (2 * gp + (k >> 1)) * (C / 2) + 2 * half + (k & 1)) & (D / 2 - 1);
                } else {
                    fq[k] = ch + k;
                }
            }
            // cos and sin of this lane's 4 frequencies in table row `row`
            auto load_row4 = [&](const float *row, float4 &cv, float4 &sv) {
                if constexpr (TQ) {
                    cv = make_float4(__ldg(row + fq[0]), __ldg(row + fq[1]), __ldg(row + fq[2]), __ldg(row + fq[3]));
                    sv = make_float4(__ldg(row + D / 2 + fq[0]), __ldg(row + D / 2 + fq[1]), __ldg(row + D / 2 + fq[2]),
                                     __ldg(row + D / 2 + fq[3]));
                } else {
                    cv = __ldg(reinterpret_cast<const float4 *>(row + ch));
                    sv = __ldg(reinterpret_cast<const float4 *>(row + D / 2 + ch));
                }
            };
            const uint32_t *idx_b = a.idx + ((size_t)b * a.Hkv + h) * (size_t)a.Nmax * NP + ((size_t)gp << 2);
            const uint32_t ring = (uint32_t)__cvta_generic_to_shared(smem) + TBL + (uint32_t)tid * 16u;

            // queue the first DEPTH iterations of this slot before staging the slices
            const int pfirst = tok_begin + slot * TT;
#pragma unroll
            for (int d = 0; d < DEPTH; ++d) {
                const int p = pfirst + d * STRIDE;
#pragma unroll
                for (int u = 0; u < NW; ++u)
                    if (p + 4 * u < tok_end)
                        cp_async16(ring + (uint32_t)(d * QB + u * NT * 16), idx_b + (size_t)((p >> 2) + u) * NP * 4);
                cp_async_commit();
            }

            const bool restage = !KEEP || h != staged_h;   // CTA-uniform
            staged_h = h;
            if (!restage) {
            } else if constexpr (!PG) {
            // stage the K and V slices as bank-private replicas (rows >= K zeroed)
            {
                const uint16_t *sk = a.slk + (size_t)h * a.K * C;
                const uint16_t *sv = a.slv + (size_t)h * a.K * C;
                for (int it = tid; it < 256 * 2 * REPL; it += NT) {
                    const int rep = it % REPL;
                    const int kv = (it / REPL) & 1;
                    const int r = it / (2 * REPL);
                    unsigned char *dst = smem + r * 256 + kv * 128 + rep * EB;
                    const uint16_t *src = (kv ? sv : sk) + (size_t)r * C;
                    if constexpr (C == 4) {
                        uint2 v = make_uint2(0u, 0u);
                        if (r < a.K) v = __ldg(reinterpret_cast<const uint2 *>(src));
                        *reinterpret_cast<uint2 *>(dst) = v;
                    } else {
#pragma unroll
                        for (int u = 0; u < EB / 16; ++u) {
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);
                            if (r < a.K) v = __ldg(reinterpret_cast<const uint4 *>(src) + u);
                            *reinterpret_cast<uint4 *>(dst + 16 * u) = v;
                        }
                    }
                }
            }

            } else {
                // code-major per-group tables (rows >= K zeroed): 16-byte chunks of every row
                constexpr int CH = D / 8;                          // chunks of one K (or V) row
                const uint4 *sk = reinterpret_cast<const uint4 *>(a.slk + (size_t)h * a.K * D);
                const uint4 *sv = reinterpret_cast<const uint4 *>(a.slv + (size_t)h * a.K * D);
                for (int it = tid; it < 256 * 2 * CH; it += NT) {
                    const int j = it % CH;
                    const int kv = (it / CH) & 1;
                    const int r = it / (2 * CH);
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (r < a.K) v = __ldg((kv ? sv : sk) + (size_t)r * CH + j);
                    if constexpr (D == 128) {
                        *reinterpret_cast<uint4 *>(smem + kv * 65536 + r * 256 + j * 16) = v;
                    } else {
                        *reinterpret_cast<uint4 *>(smem + r * 256 + kv * 128 + j * 16) = v;
                        *reinterpret_cast<uint4 *>(smem + 65536 + r * 256 + kv * 128 + ((j * 16 + 64) & 127)) = v;
                    }
                }
            }

            float2 qlo[QPK][2], qhi[QPK][2];
#pragma unroll
            for (int j = 0; j < QPK; ++j) {
                const uint16_t *qp = a.q + ((size_t)b * a.Hq + h * QPK + j) * D;
                if constexpr (TQ) {
                    // q / w at the lane's permuted pairs (a pair's two channels share their weight)
                    const float *wp = a.tw + (size_t)h * D;
                    float ql[4], qh[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float sc = a.qscale / __ldg(wp + fq[k]);
                        ql[k] = bf16_to_f32(qp[fq[k]]) * sc;
                        qh[k] = bf16_to_f32(qp[D / 2 + fq[k]]) * sc;
                    }
                    qlo[j][0] = f2(ql[0], ql[1]);
                    qlo[j][1] = f2(ql[2], ql[3]);
                    qhi[j][0] = f2(qh[0], qh[1]);
                    qhi[j][1] = f2(qh[2], qh[3]);
                } else {
                    const uint2 lo = *reinterpret_cast<const uint2 *>(qp + ch);
                    const uint2 hi = *reinterpret_cast<const uint2 *>(qp + D / 2 + ch);
                    qlo[j][0] = f2(bf16lo(lo.x) * a.qscale, bf16hi(lo.x) * a.qscale);
                    qlo[j][1] = f2(bf16lo(lo.y) * a.qscale, bf16hi(lo.y) * a.qscale);
                    qhi[j][0] = f2(bf16lo(hi.x) * a.qscale, bf16hi(hi.x) * a.qscale);
                    qhi[j][1] = f2(bf16lo(hi.y) * a.qscale, bf16hi(hi.y) * a.qscale);
                }
            }
            // one-position rotation of this lane's 4 frequencies (RoPE table row 1)
            float2 c1[2], s1[2];
            {
                float4 cv, sv;
                load_row4(a.rope + D, cv, sv);
                c1[0] = f2(cv.x, cv.y);
                c1[1] = f2(cv.z, cv.w);
                s1[0] = f2(sv.x, sv.y);
                s1[1] = f2(sv.z, sv.w);
            }
            const float2 ns1[2] = {neg2(s1[0]), neg2(s1[1])};
            const float2 tc1[2] = {f2(2.f * c1[0].x, 2.f * c1[0].y), f2(2.f * c1[1].x, 2.f * c1[1].y)};   // 2 cos(w)
            const float2 nqlo[2] = {neg2(qlo[0][0]), neg2(qlo[0][1])};
            float m_[QPK], l_[QPK];
            float2 olo[QPK][2], ohi[QPK][2];
#pragma unroll
            for (int j = 0; j < QPK; ++j) {
                m_[j] = -CUDART_INF_F;
                l_[j] = 0.f;
                olo[j][0] = olo[j][1] = ohi[j][0] = ohi[j][1] = f2(0.f, 0.f);
            }
            const int tk = tile_token<TT, NL>(ls);                 // token of the iteration this lane finishes

            // RoPE values at each iteration's first token p0.  XR: carried from the previous iteration
            // by one complex multiply with e^{-+i STRIDE w} (ROTQ: the rotated query itself), and set
            // from the table row every 16 iterations so that rounding stays within 16 products;
            // otherwise the table row is loaded one iteration ahead.
            float4 ra_c, ra_s;
            float2 xa_c[2], xa_s[2], sc[2], ssn[2];
            if constexpr (XR) {
                sc[0] = sc[1] = ssn[0] = ssn[1] = f2(0.f, 0.f);
                if (STRIDE < a.Nmax) {                       // else no slot runs a second iteration
                    float4 c4, s4;
                    load_row4(a.rope + (size_t)STRIDE * D, c4, s4);
                    sc[0] = f2(c4.x, c4.y);
                    sc[1] = f2(c4.z, c4.w);
                    ssn[0] = f2(s4.x, s4.y);
                    ssn[1] = f2(s4.z, s4.w);
                }
            } else {
                load_row4(a.rope + (size_t)min(pfirst, a.Nmax - 4) * D, ra_c, ra_s);
            }
            __syncthreads();

            int stage = 0, iter = 0;
            for (int p0 = pfirst; p0 < tok_end; p0 += STRIDE, ++iter) {
                cp_async_wait<DEPTH - 1>();                        // this thread's oldest queued stage has landed
                uint4 w4[NW];
#pragma unroll
                for (int u = 0; u < NW; ++u) {
                    const uint32_t addr = ring + (uint32_t)(stage * QB + u * NT * 16);
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w4[u].x), "=r"(w4[u].y), "=r"(w4[u].z), "=r"(w4[u].w) : "r"(addr) : "memory");
                }
                // the stage has been read into registers: queue the iteration DEPTH steps ahead into it
                {
                    const int pq = p0 + DEPTH * STRIDE;
#pragma unroll
                    for (int u = 0; u < NW; ++u)
                        if (pq + 4 * u < tok_end)
                            cp_async16(ring + (uint32_t)(stage * QB + u * NT * 16), idx_b + (size_t)((pq >> 2) + u) * NP * 4);
                    cp_async_commit();
                    stage = stage + 1 == DEPTH ? 0 : stage + 1;
                }
                float2 cs[2], sn[2];
                if constexpr (XR) {
                    if ((iter & 15) == 0) {
                        float4 c4, s4;
                        load_row4(a.rope + (size_t)min(p0, a.Nmax - 4) * D, c4, s4);
                        cs[0] = f2(c4.x, c4.y);
                        cs[1] = f2(c4.z, c4.w);
                        sn[0] = f2(s4.x, s4.y);
                        sn[1] = f2(s4.z, s4.w);
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            if constexpr (ROTQ) {
                                xa_c[i] = __ffma2_rn(qlo[0][i], cs[i], __fmul2_rn(qhi[0][i], sn[i]));
                                xa_s[i] = __ffma2_rn(qhi[0][i], cs[i], __fmul2_rn(nqlo[i], sn[i]));
                            } else {
                                xa_c[i] = cs[i];
                                xa_s[i] = sn[i];
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const float2 re = xa_c[i], im = xa_s[i];
                            if constexpr (ROTQ) {                 // times e^{-i STRIDE w}
                                xa_c[i] = __ffma2_rn(re, sc[i], __fmul2_rn(im, ssn[i]));
                                xa_s[i] = __ffma2_rn(im, sc[i], __fmul2_rn(re, neg2(ssn[i])));
                            } else {                              // times e^{+i STRIDE w}
                                xa_c[i] = __ffma2_rn(re, sc[i], __fmul2_rn(im, neg2(ssn[i])));
                                xa_s[i] = __ffma2_rn(im, sc[i], __fmul2_rn(re, ssn[i]));
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        cs[i] = xa_c[i];
                        sn[i] = xa_s[i];
                    }
                } else {
                    cs[0] = f2(ra_c.x, ra_c.y);
                    cs[1] = f2(ra_c.z, ra_c.w);
                    sn[0] = f2(ra_s.x, ra_s.y);
                    sn[1] = f2(ra_s.z, ra_s.w);
                    load_row4(a.rope + (size_t)min(p0 + STRIDE, a.Nmax - 4) * D, ra_c, ra_s);
                }

                // ---- values of the tile: gathered now and used after the softmax when registers allow
                // (one or two query heads per KV head); otherwise gathered in the value loop
                constexpr bool VEARLY = QPK <= 2;
                uint2 vraw[TT][2];
                if constexpr (VEARLY) {
#pragma unroll
                    for (int k = 0; k < TT; ++k) {
                        const uint32_t w = word_k(w4[k >> 2], k & 3);
                        vraw[k][0] = lds64(smem, __byte_perm(w, colv_lo, 0x7624));
                        vraw[k][1] = lds64(smem, __byte_perm(w, colv_hi, 0x7634));
                    }
                }

                // ---- keys: rebuild, score.  ROTQ: per pair f the term is Re(Z) k_f + Im(Z) k_{f+D/2} with
                // Z = (q_f + i q_{f+D/2}) e^{-i p w_f}, advanced along the tile (see the header).  Otherwise the
                // rebuilt keys are rotated by (cos, sin), advanced the same way, and shared by the query heads.
                float sig = 1.f;                                   // TaSQ scale of the token this lane finishes
                if constexpr (TQ) {
                    const int n = p0 + tk;
                    if (n < tok_end) sig = __half2float(__ushort_as_half(__ldg(a.tsig + (size_t)b * a.Nmax + n)));
                }
                float ps[QPK][TT];
                float2 zu[2], zw[2], xu[2], xw[2];                // X_k and X_{k-1} of the advanced pair
                if constexpr (ROTQ) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if constexpr (XR) {                   // cs, sn already hold Z
                            zu[i] = cs[i];
                            zw[i] = sn[i];
                        } else {
                            zu[i] = __ffma2_rn(qlo[0][i], cs[i], __fmul2_rn(qhi[0][i], sn[i]));
                            zw[i] = __ffma2_rn(qhi[0][i], cs[i], __fmul2_rn(nqlo[i], sn[i]));
                        }
                    }
                }
#pragma unroll
                for (int k = 0; k < TT; ++k) {
                    if (k > 0) {
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            // the pair (re, im) advanced by one position: ROTQ by e^{-iw}, else by e^{+iw}
                            float2 &re = ROTQ ? zu[i] : cs[i];
                            float2 &im = ROTQ ? zw[i] : sn[i];
                            float2 nre, nim;
                            if (k == 1) {
                                nre = ROTQ ? __ffma2_rn(re, c1[i], __fmul2_rn(im, s1[i])) : __ffma2_rn(re, c1[i], __fmul2_rn(im, ns1[i]));
                                nim = ROTQ ? __ffma2_rn(im, c1[i], __fmul2_rn(re, ns1[i])) : __ffma2_rn(im, c1[i], __fmul2_rn(re, s1[i]));
                            } else {
                                nre = __ffma2_rn(tc1[i], re, neg2(xu[i]));
                                nim = __ffma2_rn(tc1[i], im, neg2(xw[i]));
                            }
                            xu[i] = re;
                            xw[i] = im;
                            re = nre;
                            im = nim;
                        }
                    }
                    const uint32_t w = word_k(w4[k >> 2], k & 3);
                    const uint2 elo = lds64(smem, __byte_perm(w, colk_lo, 0x7604));
                    const uint2 ehi = lds64(smem, __byte_perm(w, colk_hi, 0x7614));
                    // kl: low channels (real parts) of the lane's pairs, kh: their partners (imaginary parts)
                    float2 kl[2], kh[2];
                    if constexpr (TQ) {
                        // a TaSQ entry interleaves each pair's two channels: (f, f + D/2, f', f' + D/2)
                        kl[0] = f2(bf16lo(elo.x), bf16lo(elo.y));
                        kh[0] = f2(bf16hi(elo.x), bf16hi(elo.y));
                        kl[1] = f2(bf16lo(ehi.x), bf16lo(ehi.y));
                        kh[1] = f2(bf16hi(ehi.x), bf16hi(ehi.y));
                    } else {
                        kl[0] = unpack2(elo.x);
                        kl[1] = unpack2(elo.y);
                        kh[0] = unpack2(ehi.x);
                        kh[1] = unpack2(ehi.y);
                    }
                    if constexpr (ROTQ) {
                        float2 acc = __fmul2_rn(zu[0], kl[0]);
                        acc = __ffma2_rn(zw[0], kh[0], acc);
                        acc = __ffma2_rn(zu[1], kl[1], acc);
                        acc = __ffma2_rn(zw[1], kh[1], acc);
                        ps[0][k] = acc.x + acc.y;
                    } else {
                        float2 rlo[2], rhi[2];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            rlo[i] = __ffma2_rn(kl[i], cs[i], __fmul2_rn(kh[i], neg2(sn[i])));   // kl*cos - kh*sin
                            rhi[i] = __ffma2_rn(kh[i], cs[i], __fmul2_rn(kl[i], sn[i]));         // kh*cos + kl*sin
                        }
#pragma unroll
                        for (int j = 0; j < QPK; ++j) {
                            float2 acc = __fmul2_rn(qlo[j][0], rlo[0]);
                            acc = __ffma2_rn(qhi[j][0], rhi[0], acc);
                            acc = __ffma2_rn(qlo[j][1], rlo[1], acc);
                            acc = __ffma2_rn(qhi[j][1], rhi[1], acc);
                            ps[j][k] = acc.x + acc.y;
                        }
                    }
                }

                // ---- reduce-scatter the scores over the slot, online-softmax update
                // Lazy maximum: the reference only has to stay within 2^8 of the running maximum for the
                // weights to stay finite, so it moves (with an exact rescale) only when a score of the
                // iteration exceeds it by more than 8 in log2 units.
                float pe[QPK], sc[QPK] = {};                 // sc is set below, before lazy_max runs
                auto lazy_max = [&](int j) {
                    float tmax = sc[j];
#pragma unroll
                    for (int o = NL / 2; o >= NL / TT; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(slot_mask, tmax, o));
                    const float corr = ex2(m_[j] - tmax);
                    l_[j] *= corr;
                    const float2 c2 = f2(corr, corr);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        olo[j][i] = __fmul2_rn(olo[j][i], c2);
                        ohi[j][i] = __fmul2_rn(ohi[j][i], c2);
                    }
                    m_[j] = tmax;
                };
                if constexpr (QPK == 1) {
                    float keep = reduce_scatter<TT, NL>(ps[0], ls, slot_mask);
                    if constexpr (TQ) keep *= sig;
                    sc[0] = (p0 + tk < tok_end && p0 + tk >= st) ? keep : -CUDART_INF_F;
                    if (__any_sync(slot_mask, sc[0] > m_[0] + 8.f)) lazy_max(0);
                } else {
                    // one vote covers every query head (measured 15 % faster than a vote per head at 4
                    // query heads); the rare update then checks each head
                    bool over = false;
                    const bool live = p0 + tk < tok_end && p0 + tk >= st;
#pragma unroll
                    for (int j = 0; j < QPK; ++j) {
                        float keep = reduce_scatter<TT, NL>(ps[j], ls, slot_mask);
                        if constexpr (TQ) keep *= sig;
                        sc[j] = live ? keep : -CUDART_INF_F;
                        over |= sc[j] > m_[j] + 8.f;
                    }
                    if (__any_sync(slot_mask, over)) {
#pragma unroll
                        for (int j = 0; j < QPK; ++j)
                            if (__any_sync(slot_mask, sc[j] > m_[j] + 8.f)) lazy_max(j);
                    }
                }
#pragma unroll
                for (int j = 0; j < QPK; ++j) {
                    pe[j] = ex2(sc[j] - m_[j]);
                    l_[j] += pe[j];
                }

                // ---- values: rebuild and accumulate with each token's weight
#pragma unroll
                for (int k = 0; k < TT; ++k) {
                    const int src = slot_lane0 + tile_owner<TT, NL>(k);
                    if constexpr (!VEARLY) {
                        const uint32_t w = word_k(w4[k >> 2], k & 3);
                        vraw[k][0] = lds64(smem, __byte_perm(w, colv_lo, 0x7624));
                        vraw[k][1] = lds64(smem, __byte_perm(w, colv_hi, 0x7634));
                    }
                    const uint32_t vl[2] = {vraw[k][0].x, vraw[k][0].y}, vh[2] = {vraw[k][1].x, vraw[k][1].y};
#pragma unroll
                    for (int j = 0; j < QPK; ++j) {
                        const float pk = __shfl_sync(slot_mask, pe[j], src);
                        const float2 p2 = f2(pk, pk);
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            olo[j][i] = __ffma2_rn(p2, unpack2(vl[i]), olo[j][i]);
                            ohi[j][i] = __ffma2_rn(p2, unpack2(vh[i]), ohi[j][i]);
                        }
                    }
                }
            }
            cp_async_wait<0>();

            // ---- combine the slots of this CTA, write the split's partial result
            __syncthreads();                                       // the queue (and without KEEP the slices) no longer needed
            constexpr int RS = D + 4;                              // floats per (slot, query head) record
            // l_ sums the weights of the tokens this lane finished: add the other token positions of the slot
            constexpr int TOKBITS = (TT == 8) ? 3 : 2;
            float *red = reinterpret_cast<float *>(smem + (KEEP ? REC_OFF : 0u));
#pragma unroll
            for (int j = 0; j < QPK; ++j) {
                float lsum = l_[j];
#pragma unroll
                for (int sb = 0; sb < TOKBITS; ++sb) lsum += __shfl_xor_sync(slot_mask, lsum, NL >> (1 + sb));
                float *rec = red + ((size_t)slot * QPK + j) * RS;
                *reinterpret_cast<float4 *>(rec + ch) = make_float4(olo[j][0].x, olo[j][0].y, olo[j][1].x, olo[j][1].y);
                *reinterpret_cast<float4 *>(rec + D / 2 + ch) = make_float4(ohi[j][0].x, ohi[j][0].y, ohi[j][1].x, ohi[j][1].y);
                if (ls == 0) {
                    rec[D] = m_[j];
                    rec[D + 1] = lsum;
                }
            }
            __syncthreads();
            for (int it = tid; it < QPK * D; it += NT) {
                const int d = it % D;
                const int j = it / D;
                float mx = -CUDART_INF_F;
                for (int s2 = 0; s2 < NSLOT; ++s2) mx = fmaxf(mx, red[((size_t)s2 * QPK + j) * RS + D]);
                float acc = 0.f, lsum = 0.f;
                if (mx != -CUDART_INF_F) {
                    for (int s2 = 0; s2 < NSLOT; ++s2) {
                        const float *rec = red + ((size_t)s2 * QPK + j) * RS;
                        const float wgt = ex2(rec[D] - mx);
                        acc += rec[d] * wgt;
                        lsum += rec[D + 1] * wgt;
                    }
                }
                const size_t rec = (size_t)piece * QPK + j;
                a.ws_o[rec * D + d] = acc;
                if (d == 0) a.ws_ml[rec] = f2(mx, lsum);
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
