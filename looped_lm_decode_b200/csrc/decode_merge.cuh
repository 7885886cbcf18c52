// The log-sum-exp merge of the split kernels' partial records (LoopVQ paper, Sec. 4.3 "Attention": the
// tokens are cut into splits whose partial outputs are combined through their log-sum-exp, which is
// exact), and the attention to a bf16 window folded into it.
#pragma once

#include "decode_kernel.cuh"

namespace loopvq {

// Log-sum-exp merge of the pieces of every (sequence, query head).  Launched as a programmatic
// dependent of the split kernel: it finds its segment's records while the split kernel finishes, then
// waits for that grid (griddepcontrol.wait returns once the split kernel has completed and its writes
// are visible) before reading them.  The records' (max, sum) pairs, then their outputs, are read in
// batches of independent loads.
//
// With a bf16 window (LoopVQ paper, Sec. 4.3 "Cache layout" and "Attention": the sink and recent tokens
// stay in bf16 and their attention is combined with the coded tokens' through the log-sum-exp), the
// merge first attends to the window slots [0, fill_b) itself, before the wait, so that this work
// overlaps the split kernel: warp w takes slots w, w + D/32, ..., each lane D/32 channels of a slot,
// an online softmax per warp, and the warps' results are combined in shared memory.  Window keys are
// stored rotated, so no RoPE is applied to them.  With a token to append (a.nk), slot fill_b - 1 is that
// token: every CTA reads it from the input, and the CTA of the KV group's first query head writes it into
// the window (rotated key, key before RoPE, value), which the next calls and the page roll read.
template <int D>
__global__ void __launch_bounds__(D) merge_kernel(const DecodeArgs a) {
    constexpr int RB = 8;                                  // records read per batch
    constexpr int NWARP = D / 32, CPL = D / 32;            // warps; window channels per lane
    __shared__ long long info[3];                          // Tb, Pb(b), tiles of b
    __shared__ float wrec[NWARP][D + 2];                   // window: per-warp (o, max, sum)
    const int bh = blockIdx.x;
    const int b = bh / a.Hq, hq = bh % a.Hq;
    const int qpk = a.Hq / a.Hkv, h = hq / qpk, j = hq % qpk;
    const int d = threadIdx.x;
    float mw = -CUDART_INF_F, lw = 0.f, ow = 0.f;          // the window's part for channel d
    if (a.wk != nullptr) {
        const int lane = d & 31, warp = d >> 5;
        const int n = min(max(__ldg(a.wfill + b), 0), a.W);
        float qv[CPL];
        const uint16_t *qp = a.q + (size_t)bh * D + lane * CPL;
#pragma unroll
        for (int c = 0; c < CPL; ++c) qv[c] = bf16_to_f32(__ldg(qp + c)) * a.qscale;
        const size_t row0 = ((size_t)b * a.Hkv + h) * (size_t)a.W * D + lane * CPL;
        const size_t new0 = ((size_t)b * a.Hkv + h) * D;   // the appended token's row
        const int tnew = a.nk != nullptr ? n - 1 : -1;     // its slot
        if (tnew >= 0 && j == 0) {
            const size_t dst = row0 - lane * CPL + (size_t)tnew * D;
            for (int i = d; i < D / 8; i += D) {
                reinterpret_cast<uint4 *>(a.wk_w + dst)[i] = __ldg(reinterpret_cast<const uint4 *>(a.nk + new0) + i);
                reinterpret_cast<uint4 *>(a.wkp_w + dst)[i] = __ldg(reinterpret_cast<const uint4 *>(a.nkp + new0) + i);
                reinterpret_cast<uint4 *>(a.wv_w + dst)[i] = __ldg(reinterpret_cast<const uint4 *>(a.nv + new0) + i);
            }
        }
        float m = -CUDART_INF_F, l = 0.f, o[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] = 0.f;
        for (int t = warp; t < n; t += NWARP) {
            float kv[CPL], vv[CPL];
            const bool fresh = t == tnew;
            const uint16_t *kp = fresh ? a.nk + new0 + lane * CPL : a.wk + row0 + (size_t)t * D;
            const uint16_t *vp = fresh ? a.nv + new0 + lane * CPL : a.wv + row0 + (size_t)t * D;
            if constexpr (CPL == 4) {
                const uint2 k4 = __ldg(reinterpret_cast<const uint2 *>(kp));
                const uint2 v4 = __ldg(reinterpret_cast<const uint2 *>(vp));
                kv[0] = bf16lo(k4.x); kv[1] = bf16hi(k4.x); kv[2] = bf16lo(k4.y); kv[3] = bf16hi(k4.y);
                vv[0] = bf16lo(v4.x); vv[1] = bf16hi(v4.x); vv[2] = bf16lo(v4.y); vv[3] = bf16hi(v4.y);
            } else {
                const uint32_t k2 = __ldg(reinterpret_cast<const uint32_t *>(kp));
                const uint32_t v2 = __ldg(reinterpret_cast<const uint32_t *>(vp));
                kv[0] = bf16lo(k2); kv[1] = bf16hi(k2);
                vv[0] = bf16lo(v2); vv[1] = bf16hi(v2);
            }
            float sc = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) sc = fmaf(qv[c], kv[c], sc);
#pragma unroll
            for (int o2 = 16; o2 >= 1; o2 >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o2);
            if (sc > m) {
                const float corr = ex2(m - sc);
                l *= corr;
#pragma unroll
                for (int c = 0; c < CPL; ++c) o[c] *= corr;
                m = sc;
            }
            const float pw = ex2(sc - m);
            l += pw;
#pragma unroll
            for (int c = 0; c < CPL; ++c) o[c] = fmaf(pw, vv[c], o[c]);
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) wrec[warp][lane * CPL + c] = o[c];
        if (lane == 0) {
            wrec[warp][D] = m;
            wrec[warp][D + 1] = l;
        }
    }
    if (d < 32) {
        long long Tb, Pb;
        head_tiles(a, d, b, Tb, Pb);
        int base, st, len;
        const int nt = seq_tiles(a, b, base, st, len);
        if (d == 0) {
            info[0] = Tb;
            info[1] = Pb;
            info[2] = nt;
        }
    }
    __syncthreads();
    if (a.wk != nullptr) {
#pragma unroll
        for (int w = 0; w < NWARP; ++w) mw = fmaxf(mw, wrec[w][D]);
        if (mw != -CUDART_INF_F) {
#pragma unroll
            for (int w = 0; w < NWARP; ++w) {
                const float wgt = ex2(wrec[w][D] - mw);
                ow += wrec[w][d] * wgt;
                lw += wrec[w][D + 1] * wgt;
            }
        }
    }
    const long long Tb = info[0], T = Tb * a.Hkv, G = a.ncta;
    const long long P = h * Tb + info[1], E = P + info[2];  // tiles [P, E) of segment s
    const long long s = (long long)h * a.B + b;
    long long c0 = 0, c1 = -1;
    if (E > P) {
        c0 = cta_of_tile(P, T, G);
        c1 = cta_of_tile(E - 1, T, G);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    float mx = -CUDART_INF_F, acc = 0.f, lsum = 0.f;
    for (long long cb = c0; cb <= c1; cb += RB) {
        float2 ml[RB];
        float o[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const long long c = cb + r;
            const bool live = c <= c1 && cta_first_tile(c, T, G) < cta_first_tile(c + 1, T, G);
            const size_t rec = (size_t)(s + c) * qpk + j;
            ml[r] = live ? __ldcg(a.ws_ml + rec) : make_float2(-CUDART_INF_F, 0.f);
            o[r] = live ? __ldcg(a.ws_o + rec * D + d) : 0.f;
        }
        float bm = mx;
#pragma unroll
        for (int r = 0; r < RB; ++r) bm = fmaxf(bm, ml[r].x);
        if (bm == -CUDART_INF_F) continue;
        const float corr = ex2(mx - bm);                   // 0 while mx is still -inf
        acc *= corr;
        lsum *= corr;
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const float wgt = ex2(ml[r].x - bm);           // 0 for absent records
            acc += o[r] * wgt;
            lsum += ml[r].y * wgt;
        }
        mx = bm;
    }
    if (mw != -CUDART_INF_F) {                             // fold in the window's part
        const float bm = fmaxf(mx, mw);
        const float cc = ex2(mx - bm), cw = ex2(mw - bm);
        acc = acc * cc + ow * cw;
        lsum = lsum * cc + lw * cw;
        mx = bm;
    }
    const bool any = (mx != -CUDART_INF_F) && lsum > 0.f;
    a.out[(size_t)bh * D + d] = any ? acc / lsum : 0.f;
    if (a.lse != nullptr && d == 0)
        a.lse[bh] = any ? (mx + log2f(lsum)) * 0.69314718055994530942f : -CUDART_INF_F;
}

}  // namespace loopvq
