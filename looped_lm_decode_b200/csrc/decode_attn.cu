// Decode attention over the loop-axis coded cache, one loop step of one layer.
//
// LoopVQ paper, Sec. 4.3 "Attention" and App. C: at loop step t every index is
// looked up in that step's codebook slice B_t held in shared memory, keys are
// rebuilt before RoPE and rotated from a per-position cos/sin table, and the
// quantized tokens are cut into splits processed by separate thread blocks whose
// partial outputs are merged through their log-sum-exp (exact softmax).
//
// B200 design (not the pages' kernel):
//  * One CTA per (token split, KV head, group of NBT sequences).  All sequences of
//    the group share the head's codebook slices and each RoPE table row, so a
//    row loaded into registers serves NBT sequences (App. C shares rows between
//    two requests; here NBT of them).
//  * The K and V slices are staged as bank-private replicas: entry r of the copy
//    used by lane l sits at byte r*256 + kv*128 + (l % R)*EB, EB = 2c bytes,
//    R = 128/EB lanes per shared-memory wavefront.  A gather of any 16 (c=4) or
//    8 (c=8) random entries by one half/quarter warp then hits distinct banks.
//  * A token slot of NP = D/(2c) lanes handles 4-token tiles.  Lane p owns the
//    channel groups p and p + NP, i.e. the two halves of its RoPE pairs, so a
//    lane rotates its own keys with one cos and one sin vector per token.
//  * The 4 partial scores of a tile are reduce-scattered across the slot (5
//    shuffles) so each lane finishes one token and takes one exponent.
//  * fp32 math in packed pairs (FFMA2) on sm_100.
#include <math_constants.h>

#include "loopvq_internal.cuh"

namespace loopvq {

struct DecodeArgs {
    const uint32_t *idx;     // words of (layer, block, b = 0, h = 0)
    const uint16_t *slk;     // K slices of (layer, t, h = 0): [Hkv][K][c]
    const uint16_t *slv;     // V slices of (layer, t, h = 0)
    const float *rope;       // [Nmax][D]
    const uint16_t *q;       // [B][Hq][D] bf16
    const int32_t *lens;     // [B]
    float *ws_o;             // [B][Hq][nsplit][D]  unnormalised split outputs
    float2 *ws_ml;           // [B][Hq][nsplit]     (max, sum) in log2 units
    float *out;              // [B][Hq][D]
    float *lse;              // [B][Hq] or null
    int B, Hkv, Hq, K, Nmax, max_len, split_len, nsplit;
    float qscale;            // scale * log2(e)
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int C>
struct Entry;                       // C bf16 = C/2 words
template <>
struct Entry<4> {
    uint2 v;
    __device__ __forceinline__ void load(const unsigned char *p) { v = *reinterpret_cast<const uint2 *>(p); }
    __device__ __forceinline__ uint32_t w(int i) const { return i == 0 ? v.x : v.y; }
};
template <>
struct Entry<8> {
    uint4 v;
    __device__ __forceinline__ void load(const unsigned char *p) { v = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ uint32_t w(int i) const {
        return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
    }
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 unpack2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }

template <int D, int C, int QPK, int NBT, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 3) decode_split_kernel(const DecodeArgs a) {
    constexpr int NP = D / (2 * C);         // lanes per token slot
    constexpr int SPW = 32 / NP;            // slots per warp
    constexpr int NSLOT = WARPS * SPW;
    constexpr int EB = 2 * C;               // bytes of one slice entry
    constexpr int REPL = 128 / EB;          // replicas = lanes per shared-memory wavefront
    constexpr int C2 = C / 2;               // float2 per group
    static_assert(NP >= 4 && NP <= 16, "slot width");

    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, h = blockIdx.y, b0 = blockIdx.z * NBT;
    const int tok_begin = split * a.split_len;
    const int tok_end = min(tok_begin + a.split_len, a.max_len);

    // ---- stage this head's K and V slices as bank-private replicas (rows >= K zeroed)
    {
        const uint16_t *sk = a.slk + (size_t)h * a.K * C;
        const uint16_t *sv = a.slv + (size_t)h * a.K * C;
        for (int it = tid; it < 256 * 2 * REPL; it += WARPS * 32) {
            const int rep = it % REPL;
            const int kv = (it / REPL) & 1;
            const int r = it / (2 * REPL);
            unsigned char *dst = smem + r * 256 + kv * 128 + rep * EB;
            const uint16_t *src = (kv ? sv : sk) + (size_t)r * C;
            if constexpr (C == 4) {
                uint2 v = make_uint2(0u, 0u);
                if (r < a.K) v = *reinterpret_cast<const uint2 *>(src);
                *reinterpret_cast<uint2 *>(dst) = v;
            } else {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (r < a.K) v = *reinterpret_cast<const uint4 *>(src);
                *reinterpret_cast<uint4 *>(dst) = v;
            }
        }
    }

    const int slot = warp * SPW + lane / NP;
    const int gp = lane % NP;
    const unsigned slot_mask = ((1u << NP) - 1u) << (lane & ~(NP - 1));
    const int slot_lane0 = lane & ~(NP - 1);

    int lenb[NBT];
    const uint32_t *idx_bh[NBT];
    float2 qlo[NBT][QPK][C2], qhi[NBT][QPK][C2];
#pragma unroll
    for (int bb = 0; bb < NBT; ++bb) {
        const int b = b0 + bb;
        int len = 0;
        if (b < a.B) len = min(max(a.lens[b], 0), a.max_len);
        lenb[bb] = len;
        const int bc = b < a.B ? b : 0;
        idx_bh[bb] = a.idx + ((size_t)bc * a.Hkv + h) * (size_t)a.Nmax * NP;
#pragma unroll
        for (int j = 0; j < QPK; ++j) {
            const uint16_t *qp = a.q + ((size_t)bc * a.Hq + h * QPK + j) * D;
#pragma unroll
            for (int i = 0; i < C2; ++i) {
                const uint32_t lo = *reinterpret_cast<const uint32_t *>(qp + gp * C + 2 * i);
                const uint32_t hi = *reinterpret_cast<const uint32_t *>(qp + D / 2 + gp * C + 2 * i);
                qlo[bb][j][i] = f2(bf16lo(lo) * a.qscale, bf16hi(lo) * a.qscale);
                qhi[bb][j][i] = f2(bf16lo(hi) * a.qscale, bf16hi(hi) * a.qscale);
            }
        }
    }

    float m_[NBT][QPK], l_[NBT][QPK];
    float2 olo[NBT][QPK][C2], ohi[NBT][QPK][C2];
#pragma unroll
    for (int bb = 0; bb < NBT; ++bb)
#pragma unroll
        for (int j = 0; j < QPK; ++j) {
            m_[bb][j] = -CUDART_INF_F;
            l_[bb][j] = 0.f;
#pragma unroll
            for (int i = 0; i < C2; ++i) olo[bb][j][i] = ohi[bb][j][i] = f2(0.f, 0.f);
        }

    const unsigned char *sk_lane = smem + (lane % REPL) * EB;
    const unsigned char *sv_lane = sk_lane + 128;
    const bool hb = (gp & (NP / 2)) != 0;
    const bool mb = (gp & (NP / 4)) != 0;
    const int tk = (hb ? 2 : 0) + (mb ? 1 : 0);   // token of the tile this lane finishes

    __syncthreads();

    for (int p0 = tok_begin + slot * 4; p0 < tok_end; p0 += NSLOT * 4) {
        // index words of the tile for every sequence of the group (uniform per slot)
        uint4 w4[NBT];
#pragma unroll
        for (int bb = 0; bb < NBT; ++bb)
            w4[bb] = p0 < lenb[bb]
                         ? __ldg(reinterpret_cast<const uint4 *>(idx_bh[bb] + (((size_t)(p0 >> 2) * NP + gp) << 2)))
                         : make_uint4(0u, 0u, 0u, 0u);

        // ---- keys: rebuild, rotate with this token's RoPE row, partial dot per query head
        float ps[NBT][QPK][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 cs[C2], sn[C2];
            const float *row = a.rope + (size_t)(p0 + k) * D + gp * C;
#pragma unroll
            for (int i = 0; i < C / 4; ++i) {
                const float4 cv = __ldg(reinterpret_cast<const float4 *>(row) + i);
                const float4 sv = __ldg(reinterpret_cast<const float4 *>(row + D / 2) + i);
                cs[2 * i] = f2(cv.x, cv.y);
                cs[2 * i + 1] = f2(cv.z, cv.w);
                sn[2 * i] = f2(sv.x, sv.y);
                sn[2 * i + 1] = f2(sv.z, sv.w);
            }
#pragma unroll
            for (int bb = 0; bb < NBT; ++bb) {
                const uint32_t w = k == 0 ? w4[bb].x : (k == 1 ? w4[bb].y : (k == 2 ? w4[bb].z : w4[bb].w));
                Entry<C> elo, ehi;
                elo.load(sk_lane + __byte_perm(w, 0, 0x4404));
                ehi.load(sk_lane + __byte_perm(w, 0, 0x4414));
                float2 rlo[C2], rhi[C2];
#pragma unroll
                for (int i = 0; i < C2; ++i) {
                    const float2 kl = unpack2(elo.w(i));
                    const float2 kh = unpack2(ehi.w(i));
                    const float2 khn = unpack2(ehi.w(i) ^ 0x80008000u);      // -kh
                    rlo[i] = __ffma2_rn(khn, sn[i], __fmul2_rn(kl, cs[i]));  // kl*cos - kh*sin
                    rhi[i] = __ffma2_rn(kl, sn[i], __fmul2_rn(kh, cs[i]));   // kh*cos + kl*sin
                }
#pragma unroll
                for (int j = 0; j < QPK; ++j) {
                    float2 acc = __fmul2_rn(qlo[bb][j][0], rlo[0]);
                    acc = __ffma2_rn(qhi[bb][j][0], rhi[0], acc);
#pragma unroll
                    for (int i = 1; i < C2; ++i) {
                        acc = __ffma2_rn(qlo[bb][j][i], rlo[i], acc);
                        acc = __ffma2_rn(qhi[bb][j][i], rhi[i], acc);
                    }
                    ps[bb][j][k] = acc.x + acc.y;
                }
            }
        }

        // ---- reduce-scatter the 4 scores over the slot, online-softmax update
        float pe[NBT][QPK];
#pragma unroll
        for (int bb = 0; bb < NBT; ++bb) {
            const int len = lenb[bb];
#pragma unroll
            for (int j = 0; j < QPK; ++j) {
                pe[bb][j] = 0.f;
                if (p0 >= len) continue;                   // uniform within the slot
                float keep0 = hb ? ps[bb][j][2] : ps[bb][j][0], keep1 = hb ? ps[bb][j][3] : ps[bb][j][1];
                const float send0 = hb ? ps[bb][j][0] : ps[bb][j][2], send1 = hb ? ps[bb][j][1] : ps[bb][j][3];
                keep0 += __shfl_xor_sync(slot_mask, send0, NP / 2);
                keep1 += __shfl_xor_sync(slot_mask, send1, NP / 2);
                float keep = mb ? keep1 : keep0;
                const float send = mb ? keep0 : keep1;
                keep += __shfl_xor_sync(slot_mask, send, NP / 4);
#pragma unroll
                for (int o = NP / 8; o >= 1; o >>= 1) keep += __shfl_xor_sync(slot_mask, keep, o);

                const float s = (p0 + tk < len) ? keep : -CUDART_INF_F;
                float tmax = fmaxf(s, __shfl_xor_sync(slot_mask, s, NP / 4));
                tmax = fmaxf(tmax, __shfl_xor_sync(slot_mask, tmax, NP / 2));
                if (tmax > m_[bb][j]) {
                    const float corr = ex2(m_[bb][j] - tmax);
                    l_[bb][j] *= corr;
                    const float2 c2 = f2(corr, corr);
#pragma unroll
                    for (int i = 0; i < C2; ++i) {
                        olo[bb][j][i] = __fmul2_rn(olo[bb][j][i], c2);
                        ohi[bb][j][i] = __fmul2_rn(ohi[bb][j][i], c2);
                    }
                    m_[bb][j] = tmax;
                }
                pe[bb][j] = ex2(s - m_[bb][j]);
                l_[bb][j] += pe[bb][j];
            }
        }

        // ---- values: rebuild and accumulate with each token's weight
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int src = slot_lane0 + (k >> 1) * (NP / 2) + (k & 1) * (NP / 4);
#pragma unroll
            for (int bb = 0; bb < NBT; ++bb) {
                if (p0 >= lenb[bb]) continue;               // uniform within the slot
                const uint32_t w = k == 0 ? w4[bb].x : (k == 1 ? w4[bb].y : (k == 2 ? w4[bb].z : w4[bb].w));
                Entry<C> vlo, vhi;
                vlo.load(sv_lane + __byte_perm(w, 0, 0x4424));
                vhi.load(sv_lane + __byte_perm(w, 0, 0x4434));
#pragma unroll
                for (int j = 0; j < QPK; ++j) {
                    const float pk = __shfl_sync(slot_mask, pe[bb][j], src);
                    const float2 p2 = f2(pk, pk);
#pragma unroll
                    for (int i = 0; i < C2; ++i) {
                        olo[bb][j][i] = __ffma2_rn(p2, unpack2(vlo.w(i)), olo[bb][j][i]);
                        ohi[bb][j][i] = __ffma2_rn(p2, unpack2(vhi.w(i)), ohi[bb][j][i]);
                    }
                }
            }
        }
    }

    // ---- combine the slots of this CTA, write the split's partial result
    __syncthreads();                                       // slices no longer needed
    constexpr int RS = D + 2;                              // floats per (slot, b, j) record
    float *red = reinterpret_cast<float *>(smem);
#pragma unroll
    for (int bb = 0; bb < NBT; ++bb)
#pragma unroll
        for (int j = 0; j < QPK; ++j) {
            float ls = l_[bb][j] + __shfl_xor_sync(slot_mask, l_[bb][j], NP / 4);
            ls += __shfl_xor_sync(slot_mask, ls, NP / 2);
            float *rec = red + ((size_t)(slot * NBT + bb) * QPK + j) * RS;
#pragma unroll
            for (int i = 0; i < C2; ++i) {
                rec[gp * C + 2 * i] = olo[bb][j][i].x;
                rec[gp * C + 2 * i + 1] = olo[bb][j][i].y;
                rec[D / 2 + gp * C + 2 * i] = ohi[bb][j][i].x;
                rec[D / 2 + gp * C + 2 * i + 1] = ohi[bb][j][i].y;
            }
            if (gp == 0) {
                rec[D] = m_[bb][j];
                rec[D + 1] = ls;
            }
        }
    __syncthreads();
    for (int it = tid; it < NBT * QPK * D; it += WARPS * 32) {
        const int d = it % D;
        const int j = (it / D) % QPK;
        const int bb = it / (D * QPK);
        const int b = b0 + bb;
        if (b >= a.B) continue;
        float mx = -CUDART_INF_F;
        for (int s = 0; s < NSLOT; ++s) mx = fmaxf(mx, red[((size_t)(s * NBT + bb) * QPK + j) * RS + D]);
        float acc = 0.f, lsum = 0.f;
        if (mx != -CUDART_INF_F) {
            for (int s = 0; s < NSLOT; ++s) {
                const float *rec = red + ((size_t)(s * NBT + bb) * QPK + j) * RS;
                const float wgt = ex2(rec[D] - mx);
                acc += rec[d] * wgt;
                lsum += rec[D + 1] * wgt;
            }
        }
        const size_t bh = (size_t)b * a.Hq + h * QPK + j;
        a.ws_o[(bh * a.nsplit + split) * D + d] = acc;
        if (d == 0) a.ws_ml[bh * a.nsplit + split] = f2(mx, lsum);
    }
}

// Log-sum-exp merge of the splits of every (sequence, query head).
template <int D>
__global__ void __launch_bounds__(D) merge_kernel(const DecodeArgs a) {
    const int bh = blockIdx.x;
    const int b = bh / a.Hq;
    const int d = threadIdx.x;
    const int len = min(max(a.lens[b], 0), a.max_len);
    const int ns = len > 0 ? (len + a.split_len - 1) / a.split_len : 0;
    const float2 *ml = a.ws_ml + (size_t)bh * a.nsplit;
    float mx = -CUDART_INF_F;
    for (int s = 0; s < ns; ++s) mx = fmaxf(mx, ml[s].x);
    float acc = 0.f, lsum = 0.f;
    if (mx != -CUDART_INF_F) {
        const float *o = a.ws_o + (size_t)bh * a.nsplit * D + d;
        for (int s = 0; s < ns; ++s) {
            const float wgt = ex2(ml[s].x - mx);
            acc += o[(size_t)s * D] * wgt;
            lsum += ml[s].y * wgt;
        }
    }
    const bool any = (mx != -CUDART_INF_F) && lsum > 0.f;
    a.out[(size_t)bh * D + d] = any ? acc / lsum : 0.f;
    if (a.lse != nullptr && d == 0)
        a.lse[bh] = any ? (mx + log2f(lsum)) * 0.69314718055994530942f : -CUDART_INF_F;
}

// ------------------------------------------------------------------ host side

static constexpr int kWarps = 4;

static int nbt_for(int qpk, int B) {
    int n = qpk == 1 ? 4 : (qpk == 2 ? 2 : 1);
    while (n > 1 && n / 2 >= B) n /= 2;
    return n;
}

DecodePlan plan_decode(const loopvq_cache &cc, int max_len) {
    DecodePlan p{};
    const int qpk = cc.Hq / cc.Hkv;
    const int NP = cc.D / (2 * cc.c);
    const int nslot = kWarps * (32 / NP);
    p.nbt = nbt_for(qpk, cc.B);
    p.nchunk = (cc.B + p.nbt - 1) / p.nbt;
    const int min_split = 4 * nslot;                     // one tile per slot
    const long units = (long)cc.Hkv * p.nchunk;
    const long target_ctas = 148L * 3 * 4;               // about four waves of resident CTAs
    long want = (target_ctas + units - 1) / units;
    if (want < 1) want = 1;
    long sl = max_len > 0 ? ((long)max_len + want - 1) / want : min_split;
    sl = ((sl + min_split - 1) / min_split) * min_split;
    if (sl < min_split) sl = min_split;
    p.split_len = (int)sl;
    p.nsplit = max_len > 0 ? (int)((max_len + sl - 1) / sl) : 0;
    const size_t o_bytes = (size_t)cc.B * cc.Hq * (size_t)p.nsplit * cc.D * sizeof(float);
    const size_t ml_bytes = (size_t)cc.B * cc.Hq * (size_t)p.nsplit * sizeof(float2);
    p.ws_bytes = ((o_bytes + 255) & ~(size_t)255) + ml_bytes;
    return p;
}

template <int D, int C, int QPK, int NBT>
static cudaError_t launch_t(const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    constexpr int NP = D / (2 * C);
    constexpr int NSLOT = kWarps * (32 / NP);
    const size_t red = (size_t)NSLOT * NBT * QPK * (D + 2) * sizeof(float);
    const size_t smem = red > 65536 ? red : 65536;
    auto kern = decode_split_kernel<D, C, QPK, NBT, kWarps>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (plan.nsplit > 0) {
        dim3 grid(plan.nsplit, a.Hkv, plan.nchunk);
        kern<<<grid, kWarps * 32, smem, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    merge_kernel<D><<<a.B * a.Hq, D, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D, int C>
static cudaError_t dispatch_qpk(int qpk, int nbt, const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    switch (qpk) {
        case 1:
            if (nbt == 4) return launch_t<D, C, 1, 4>(a, plan, s);
            if (nbt == 2) return launch_t<D, C, 1, 2>(a, plan, s);
            return launch_t<D, C, 1, 1>(a, plan, s);
        case 2:
            if (nbt == 2) return launch_t<D, C, 2, 2>(a, plan, s);
            return launch_t<D, C, 2, 1>(a, plan, s);
        case 4: return launch_t<D, C, 4, 1>(a, plan, s);
        case 8: return launch_t<D, C, 8, 1>(a, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const loopvq_cache &cc, const DecodePlan &plan, int layer, int t,
                          const uint16_t *q, const int32_t *lens, int max_len, float scale,
                          float *out, float *lse, void *workspace, cudaStream_t s) {
    DecodeArgs a{};
    const int beta = t / cc.Tc;
    a.idx = cc.idx + idx_base(cc, layer, beta, 0, 0);
    a.slk = cc.slices + slice_base(cc, layer, t, 0, 0);
    a.slv = cc.slices + slice_base(cc, layer, t, 1, 0);
    a.rope = cc.rope;
    a.q = q;
    a.lens = lens;
    const size_t o_bytes = (size_t)cc.B * cc.Hq * (size_t)plan.nsplit * cc.D * sizeof(float);
    a.ws_o = reinterpret_cast<float *>(workspace);
    a.ws_ml = reinterpret_cast<float2 *>(reinterpret_cast<char *>(workspace) + ((o_bytes + 255) & ~(size_t)255));
    a.out = out;
    a.lse = lse;
    a.B = cc.B;
    a.Hkv = cc.Hkv;
    a.Hq = cc.Hq;
    a.K = cc.K;
    a.Nmax = cc.Nmax;
    a.max_len = max_len;
    a.split_len = plan.split_len;
    a.nsplit = plan.nsplit;
    a.qscale = scale * 1.44269504088896340736f;
    const int qpk = cc.Hq / cc.Hkv;
    if (cc.D == 128 && cc.c == 4) return dispatch_qpk<128, 4>(qpk, plan.nbt, a, plan, s);
    if (cc.D == 128 && cc.c == 8) return dispatch_qpk<128, 8>(qpk, plan.nbt, a, plan, s);
    if (cc.D == 64 && cc.c == 4) return dispatch_qpk<64, 4>(qpk, plan.nbt, a, plan, s);
    if (cc.D == 64 && cc.c == 8) return dispatch_qpk<64, 8>(qpk, plan.nbt, a, plan, s);
    return cudaErrorInvalidValue;
}

}  // namespace loopvq
