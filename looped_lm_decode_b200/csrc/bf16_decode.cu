// Decode attention over a bf16 KV cache, and the two-part log-sum-exp merge.
//
// LoopVQ paper, Sec. 4.3 "Cache layout" and "Attention": the sink and recent
// tokens stay in bf16 and one kernel attends to them while another attends to
// the quantized tokens; their results are combined through the log-sum-exp.
// Sec. 5.3 compares LoopVQ decode against a cache held entirely in bf16; this
// kernel is that comparison on B200, at the same shapes.
//
// Design (B200): the bf16 cache is read once from HBM at 512 bytes per token
// and KV head (D = 128), so the kernel is a stream.  One CTA per (token split,
// KV head, sequence); token slots of D/8 lanes, each lane owning 8 contiguous
// channels (16 bytes of a key row and 16 of a value row).  Every thread keeps
// a DEPTH-deep queue of its own 16-byte cp.async copies (it reads back only
// what it copied, so no barrier or wait on other threads is involved); copies
// of tokens past the split end are zero-filled instead of read.  Scores are
// reduce-scattered over the slot, the softmax keeps a lazy maximum, and the
// slots of a CTA are combined in shared memory as in the coded kernel.
// Keys in the cache are already rotated (RoPE at write time), so no rotation
// happens here.
#include "decode_kernel.cuh"

namespace loopvq {

struct Bf16Args {
    const uint16_t *k, *v;   // [B][Hkv][Nmax][D]
    const uint16_t *q;       // [B][Hq][D]
    const int32_t *starts;   // [B] or null
    const int32_t *lens;     // [B]
    float *ws_o;             // [B][Hq][nsplit][D]
    float2 *ws_ml;           // [B][Hq][nsplit]
    int B, Hkv, Hq, Nmax, max_len, split_len, nsplit;
    float qscale;            // scale * log2(e)
};

// 16-byte copy that reads src_bytes (16 or 0) and zero-fills the rest
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst_smem, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void unpack8(const uint4 &w, float2 (&x)[4]) {
    x[0] = unpack2(w.x);
    x[1] = unpack2(w.y);
    x[2] = unpack2(w.z);
    x[3] = unpack2(w.w);
}

template <int D, int QPK, int WARPS, int MINB, int DEPTH>
__global__ void __launch_bounds__(WARPS * 32, MINB) bf16_split_kernel(const Bf16Args a) {
    constexpr int NL = D / 8;                              // lanes per token slot
    constexpr int SPW = 32 / NL;
    constexpr int NSLOT = WARPS * SPW;
    constexpr int NT = WARPS * 32;
    constexpr int TT = 4;                                  // tokens per slot iteration
    constexpr int STRIDE = NSLOT * TT;
    constexpr int CHUNKS = 2 * TT;                         // 16-byte copies per thread per stage (K then V)
    constexpr uint32_t QB = (uint32_t)NT * 16u * CHUNKS;   // bytes of one queue stage
    static_assert(NL >= 8 && NL <= 16, "slot width");

    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int len = min(max(__ldg(a.lens + b), 0), a.max_len);
    const int st = a.starts ? min(max(__ldg(a.starts + b), 0), len) : 0;
    const int tok_begin = (st & ~3) + split * a.split_len;  // same split convention as the coded kernel
    if (tok_begin >= len) return;
    const int tok_end = min(tok_begin + a.split_len, len);

    const int ls = lane % NL;
    const int slot = warp * SPW + lane / NL;
    const unsigned slot_mask = ((1u << NL) - 1u) << (lane & ~(NL - 1));
    const int slot_lane0 = lane & ~(NL - 1);
    const int ch = ls * 8;                                 // first of this lane's 8 channels
    const size_t row0 = ((size_t)b * a.Hkv + h) * (size_t)a.Nmax;
    const uint16_t *kb = a.k + row0 * D + ch;
    const uint16_t *vb = a.v + row0 * D + ch;
    const uint32_t ring = (uint32_t)__cvta_generic_to_shared(smem) + (uint32_t)tid * 16u;

    // copies of the iteration whose first token is p into stage `stg`: chunk j < TT is the key of token
    // p + j, chunk TT + j its value; chunk j of thread i sits at (j * NT + i) * 16, so that the 8
    // threads of a quarter warp read consecutive 16-byte words
    auto issue = [&](int p, int stg) {
#pragma unroll
        for (int j = 0; j < TT; ++j) {
            const int n = p + j;
            const bool ok = n < tok_end;
            const size_t off = (size_t)(ok ? n : tok_begin) * D;
            const uint32_t dst = ring + (uint32_t)stg * QB + (uint32_t)(j * NT) * 16u;
            cp_async16_zfill(dst, kb + off, ok ? 16u : 0u);
            cp_async16_zfill(dst + (uint32_t)(TT * NT) * 16u, vb + off, ok ? 16u : 0u);
        }
        cp_async_commit();
    };

    const int pfirst = tok_begin + slot * TT;
#pragma unroll
    for (int d = 0; d < DEPTH; ++d) issue(pfirst + d * STRIDE, d);

    float2 qv[QPK][4];
#pragma unroll
    for (int j = 0; j < QPK; ++j) {
        const uint4 w = *reinterpret_cast<const uint4 *>(a.q + ((size_t)b * a.Hq + h * QPK + j) * D + ch);
        float2 x[4];
        unpack8(w, x);
#pragma unroll
        for (int i = 0; i < 4; ++i) qv[j][i] = __fmul2_rn(x[i], f2(a.qscale, a.qscale));
    }
    float m_[QPK], l_[QPK];
    float2 o[QPK][4];
#pragma unroll
    for (int j = 0; j < QPK; ++j) {
        m_[j] = -CUDART_INF_F;
        l_[j] = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) o[j][i] = f2(0.f, 0.f);
    }
    const int tk = tile_token<TT, NL>(ls);

    int stage = 0;
    for (int p0 = pfirst; p0 < tok_end; p0 += STRIDE) {
        cp_async_wait<DEPTH - 1>();                        // this thread's oldest stage has landed
        uint4 kw[TT], vw[TT];
#pragma unroll
        for (int j = 0; j < TT; ++j) {
            const uint32_t addr = ring + (uint32_t)stage * QB + (uint32_t)(j * NT) * 16u;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(kw[j].x), "=r"(kw[j].y), "=r"(kw[j].z), "=r"(kw[j].w) : "r"(addr) : "memory");
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(vw[j].x), "=r"(vw[j].y), "=r"(vw[j].z), "=r"(vw[j].w)
                         : "r"(addr + (uint32_t)(TT * NT) * 16u)
                         : "memory");
        }
        issue(p0 + DEPTH * STRIDE, stage);                 // the stage is in registers: refill it
        stage = stage + 1 == DEPTH ? 0 : stage + 1;

        // ---- scores of the tile's tokens for every query head of this KV head
        float ps[QPK][TT];
#pragma unroll
        for (int j = 0; j < TT; ++j) {
            float2 kx[4];
            unpack8(kw[j], kx);
#pragma unroll
            for (int hq = 0; hq < QPK; ++hq) {
                float2 acc = __fmul2_rn(qv[hq][0], kx[0]);
                acc = __ffma2_rn(qv[hq][1], kx[1], acc);
                acc = __ffma2_rn(qv[hq][2], kx[2], acc);
                acc = __ffma2_rn(qv[hq][3], kx[3], acc);
                ps[hq][j] = acc.x + acc.y;
            }
        }

        // ---- reduce-scatter over the slot, online softmax with a lazy maximum (see the coded kernel)
        float pe[QPK];
#pragma unroll
        for (int hq = 0; hq < QPK; ++hq) {
            const float keep = reduce_scatter<TT, NL>(ps[hq], ls, slot_mask);
            const int n = p0 + tk;
            const float s = (n < tok_end && n >= st) ? keep : -CUDART_INF_F;
            if (__any_sync(slot_mask, s > m_[hq] + 8.f)) {
                float tmax = s;
#pragma unroll
                for (int off = NL / 2; off >= NL / TT; off >>= 1)
                    tmax = fmaxf(tmax, __shfl_xor_sync(slot_mask, tmax, off));
                const float corr = ex2(m_[hq] - tmax);
                l_[hq] *= corr;
                const float2 c2 = f2(corr, corr);
#pragma unroll
                for (int i = 0; i < 4; ++i) o[hq][i] = __fmul2_rn(o[hq][i], c2);
                m_[hq] = tmax;
            }
            pe[hq] = ex2(s - m_[hq]);
            l_[hq] += pe[hq];
        }

        // ---- values
#pragma unroll
        for (int j = 0; j < TT; ++j) {
            const int src = slot_lane0 + tile_owner<TT, NL>(j);
            float2 vx[4];
            unpack8(vw[j], vx);
#pragma unroll
            for (int hq = 0; hq < QPK; ++hq) {
                const float pk = __shfl_sync(slot_mask, pe[hq], src);
                const float2 p2 = f2(pk, pk);
#pragma unroll
                for (int i = 0; i < 4; ++i) o[hq][i] = __ffma2_rn(p2, vx[i], o[hq][i]);
            }
        }
    }
    cp_async_wait<0>();

    // ---- combine the slots of this CTA, write the split's partial result
    __syncthreads();
    constexpr int RS = D + 4;
    float *red = reinterpret_cast<float *>(smem);
#pragma unroll
    for (int hq = 0; hq < QPK; ++hq) {
        float lsum = l_[hq];
#pragma unroll
        for (int sb = 0; sb < 2; ++sb) lsum += __shfl_xor_sync(slot_mask, lsum, NL >> (1 + sb));
        float *rec = red + ((size_t)slot * QPK + hq) * RS;
        *reinterpret_cast<float4 *>(rec + ch) = make_float4(o[hq][0].x, o[hq][0].y, o[hq][1].x, o[hq][1].y);
        *reinterpret_cast<float4 *>(rec + ch + 4) = make_float4(o[hq][2].x, o[hq][2].y, o[hq][3].x, o[hq][3].y);
        if (ls == 0) {
            rec[D] = m_[hq];
            rec[D + 1] = lsum;
        }
    }
    __syncthreads();
    for (int it = tid; it < QPK * D; it += NT) {
        const int d = it % D;
        const int hq = it / D;
        float mx = -CUDART_INF_F;
        for (int s2 = 0; s2 < NSLOT; ++s2) mx = fmaxf(mx, red[((size_t)s2 * QPK + hq) * RS + D]);
        float acc = 0.f, lsum = 0.f;
        if (mx != -CUDART_INF_F) {
            for (int s2 = 0; s2 < NSLOT; ++s2) {
                const float *rec = red + ((size_t)s2 * QPK + hq) * RS;
                const float wgt = ex2(rec[D] - mx);
                acc += rec[d] * wgt;
                lsum += rec[D + 1] * wgt;
            }
        }
        const size_t bh = (size_t)b * a.Hq + h * QPK + hq;
        a.ws_o[(bh * a.nsplit + split) * D + d] = acc;
        if (d == 0) a.ws_ml[bh * a.nsplit + split] = f2(mx, lsum);
    }
}

// Two-part log-sum-exp merge: one CTA per row, D threads.  Both log-sum-exps are read before any
// thread writes, so the outputs may alias the inputs.
template <int D>
__global__ void __launch_bounds__(D) merge2_kernel(const float *out_a, const float *lse_a, const float *out_b,
                                                   const float *lse_b, float *out, float *lse) {
    const size_t r = blockIdx.x;
    const int d = threadIdx.x;
    const float la = lse_a[r], lb = lse_b[r];
    const float xa = out_a[r * D + d], xb = out_b[r * D + d];
    __syncthreads();
    const float m = fmaxf(la, lb);
    float res = 0.f, l = -CUDART_INF_F;
    if (m != -CUDART_INF_F) {
        const float wa = expf(la - m), wb = expf(lb - m);    // exp(-inf) = 0 for an empty part
        const float wsum = wa + wb;
        res = (wa * xa + wb * xb) / wsum;
        l = m + logf(wsum);
    }
    out[r * D + d] = res;
    if (lse != nullptr && d == 0) lse[r] = l;
}

// ------------------------------------------------------------------ host side

// Log-sum-exp merge of the splits of every (sequence, query head).
template <int D>
__global__ void __launch_bounds__(D) bf16_merge_kernel(const Bf16Args a, float *out, float *lse) {
    const int bh = blockIdx.x;
    const int b = bh / a.Hq;
    const int d = threadIdx.x;
    const int len = min(max(a.lens[b], 0), a.max_len);
    const int st = min(max(a.starts ? a.starts[b] : 0, 0), len);
    const int span = len - (st & ~3);                      // tokens covered by the splits
    const int ns = len > st ? (span + a.split_len - 1) / a.split_len : 0;
    const float2 *ml = a.ws_ml + (size_t)bh * a.nsplit;
    float mx = -CUDART_INF_F;
    for (int sp = 0; sp < ns; ++sp) mx = fmaxf(mx, ml[sp].x);
    float acc = 0.f, lsum = 0.f;
    if (mx != -CUDART_INF_F) {
        const float *o = a.ws_o + (size_t)bh * a.nsplit * D + d;
        for (int sp = 0; sp < ns; ++sp) {
            const float wgt = ex2(ml[sp].x - mx);
            acc += o[(size_t)sp * D] * wgt;
            lsum += ml[sp].y * wgt;
        }
    }
    const bool any = (mx != -CUDART_INF_F) && lsum > 0.f;
    out[(size_t)bh * D + d] = any ? acc / lsum : 0.f;
    if (lse != nullptr && d == 0) lse[bh] = any ? (mx + log2f(lsum)) * 0.69314718055994530942f : -CUDART_INF_F;
}

static constexpr int kBfWarps = 8;
static constexpr int kBfMinBlocks = 2;
static constexpr int kBfDepth = 3;
static constexpr long kBfTargetCtas = 148L * 2 * 4;

static size_t bf16_smem_bytes() { return (size_t)kBfDepth * kBfWarps * 32 * 16 * 8; }

DecodePlan plan_bf16(const loopvq_bf16_cache &c, int max_len) {
    DecodePlan p{};
    const int stride = 4 * kBfWarps * (32 / (c.D / 8));
    p.nbt = 1;
    p.nchunk = c.B;
    const long units = (long)c.Hkv * c.B;
    long sl = max_len > 0 ? ((long)max_len * units + kBfTargetCtas - 1) / kBfTargetCtas : stride;
    sl = ((sl + stride - 1) / stride) * stride;
    if (sl < stride) sl = stride;
    if (sl > 8192) sl = 8192;
    p.split_len = (int)sl;
    p.nsplit = max_len > 0 ? (int)((max_len + sl - 1) / sl) : 0;
    const size_t o_bytes = (size_t)c.B * c.Hq * (size_t)p.nsplit * c.D * sizeof(float);
    const size_t ml_bytes = (size_t)c.B * c.Hq * (size_t)p.nsplit * sizeof(float2);
    p.ws_bytes = ((o_bytes + 255) & ~(size_t)255) + ml_bytes;
    return p;
}

template <int D, int QPK>
static cudaError_t launch_bf16_t(const Bf16Args &a, float *out, float *lse, cudaStream_t s) {
    constexpr int NSLOT = kBfWarps * (32 / (D / 8));
    const size_t smem = bf16_smem_bytes();
    if ((size_t)NSLOT * QPK * (D + 4) * sizeof(float) > smem) return cudaErrorInvalidConfiguration;
    auto kern = bf16_split_kernel<D, QPK, kBfWarps, kBfMinBlocks, kBfDepth>;
    cudaError_t e = ensure_dynamic_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    if (a.nsplit > 0) {
        kern<<<dim3(a.nsplit, a.Hkv, a.B), kBfWarps * 32, smem, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    bf16_merge_kernel<D><<<a.B * a.Hq, D, 0, s>>>(a, out, lse);
    return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_bf16(int qpk, const Bf16Args &a, float *out, float *lse, cudaStream_t s) {
    switch (qpk) {
        case 1: return launch_bf16_t<D, 1>(a, out, lse, s);
        case 2: return launch_bf16_t<D, 2>(a, out, lse, s);
        case 4: return launch_bf16_t<D, 4>(a, out, lse, s);
        case 8: return launch_bf16_t<D, 8>(a, out, lse, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_bf16_decode(const loopvq_bf16_cache &c, const DecodePlan &plan, const uint16_t *q,
                               const int32_t *starts, const int32_t *lens, int max_len, float scale, float *out,
                               float *lse, void *workspace, cudaStream_t s) {
    Bf16Args a{};
    a.k = c.k;
    a.v = c.v;
    a.q = q;
    a.starts = starts;
    a.lens = lens;
    const size_t o_bytes = (size_t)c.B * c.Hq * (size_t)plan.nsplit * c.D * sizeof(float);
    a.ws_o = reinterpret_cast<float *>(workspace);
    a.ws_ml = reinterpret_cast<float2 *>(reinterpret_cast<char *>(workspace) + ((o_bytes + 255) & ~(size_t)255));
    a.B = c.B;
    a.Hkv = c.Hkv;
    a.Hq = c.Hq;
    a.Nmax = c.Nmax;
    a.max_len = max_len;
    a.split_len = plan.split_len;
    a.nsplit = plan.nsplit;
    a.qscale = scale * 1.44269504088896340736f;
    const int qpk = c.Hq / c.Hkv;
    if (c.D == 128) return dispatch_bf16<128>(qpk, a, out, lse, s);
    if (c.D == 64) return dispatch_bf16<64>(qpk, a, out, lse, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_merge2(const float *out_a, const float *lse_a, const float *out_b, const float *lse_b, int rows,
                          int D, float *out, float *lse, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    if (D == 128) merge2_kernel<128><<<rows, 128, 0, s>>>(out_a, lse_a, out_b, lse_b, out, lse);
    else if (D == 64) merge2_kernel<64><<<rows, 64, 0, s>>>(out_a, lse_a, out_b, lse_b, out, lse);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace loopvq
