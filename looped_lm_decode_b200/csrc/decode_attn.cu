// Decode attention over the loop-axis coded cache, one loop step of one layer:
// launch planning and dispatch.  The kernels are in decode_kernel.cuh.
//
// LoopVQ paper, Sec. 4.3 "Attention": the quantized tokens are divided into
// splits processed by separate thread blocks, and the partial outputs of all
// splits are combined using the log-sum-exp of their scores.
#include "decode_kernel.cuh"

namespace loopvq {

// ------------------------------------------------------------------ host side
//
// One CTA per (token split, KV head, sequence): 8 warps, two CTAs per SM (64 KB of codebook-slice
// replicas plus a 16 KB prefetch queue each), splits sized for about six waves of resident CTAs.

static constexpr int kWarps = 8;
static constexpr int kMinBlocks = 2;
static constexpr int kDepth = 4;
static constexpr int kWords = 1;                          // index words per lane per iteration (4-token tiles)
static constexpr long kTargetCtas = 148L * 2 * 4;
// one codebook per channel group: 128 KiB of tables, so one CTA of 16 warps per SM
static constexpr int kPgWarps = 16;
static constexpr int kPgMinBlocks = 1;
static constexpr long kPgTargetCtas = 148L * 1 * 4;

static size_t ring_smem_bytes(bool pg) {
    return (pg ? 131072 : 65536) + (size_t)kDepth * (pg ? kPgWarps : kWarps) * 32 * 16 * kWords;
}

DecodePlan plan_decode(const loopvq_cache &cc, int max_len) {
    DecodePlan p{};
    const bool pg = ncb_of(cc) > 1;
    const int warps = pg ? kPgWarps : kWarps;
    const long target = pg ? kPgTargetCtas : kTargetCtas;
    const int stride = 4 * kWords * warps * (32 / (cc.D / 8));   // tokens between two iterations of a slot
    p.nbt = 1;
    p.nchunk = cc.B;
    const long units = (long)cc.Hkv * cc.B;
    long sl = max_len > 0 ? ((long)max_len * units + target - 1) / target : stride;
    sl = ((sl + stride - 1) / stride) * stride;
    if (sl < stride) sl = stride;
    if (sl > 8192) sl = 8192;
    p.split_len = (int)sl;
    p.nsplit = max_len > 0 ? (int)((max_len + sl - 1) / sl) : 0;
    const size_t o_bytes = (size_t)cc.B * cc.Hq * (size_t)p.nsplit * cc.D * sizeof(float);
    const size_t ml_bytes = (size_t)cc.B * cc.Hq * (size_t)p.nsplit * sizeof(float2);
    p.ws_bytes = ((o_bytes + 255) & ~(size_t)255) + ml_bytes;
    return p;
}

template <int D, int C, int QPK, bool PG, bool TQ = false>
static cudaError_t launch_t(const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    constexpr int W = PG ? kPgWarps : kWarps;
    constexpr int NSLOT = W * (32 / (D / 8));
    const size_t red = (size_t)NSLOT * QPK * (D + 4) * sizeof(float);
    const size_t smem = ring_smem_bytes(PG);
    if (red > smem) return cudaErrorInvalidConfiguration;   // the slot records reuse slices and queue
    auto kern = decode_split_kernel<D, C, QPK, W, PG ? kPgMinBlocks : kMinBlocks, kDepth, kWords, PG, TQ>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (plan.nsplit > 0) {
        dim3 grid(plan.nsplit, a.Hkv, a.B);
        kern<<<grid, W * 32, smem, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    merge_kernel<D><<<a.B * a.Hq, D, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D, int C, bool PG>
static cudaError_t dispatch_qpk(int qpk, const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    switch (qpk) {
        case 1: return launch_t<D, C, 1, PG>(a, plan, s);
        case 2: return launch_t<D, C, 2, PG>(a, plan, s);
        case 4: return launch_t<D, C, 4, PG>(a, plan, s);
        case 8: return launch_t<D, C, 8, PG>(a, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int D, int C>
static cudaError_t dispatch_tq_qpk(int qpk, const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    switch (qpk) {
        case 1: return launch_t<D, C, 1, false, true>(a, plan, s);
        case 2: return launch_t<D, C, 2, false, true>(a, plan, s);
        case 4: return launch_t<D, C, 4, false, true>(a, plan, s);
        case 8: return launch_t<D, C, 8, false, true>(a, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int D, bool PG>
static cudaError_t dispatch_c(int c, int qpk, const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    switch (c) {
        case 4: return dispatch_qpk<D, 4, PG>(qpk, a, plan, s);
        case 8: return dispatch_qpk<D, 8, PG>(qpk, a, plan, s);
        case 16: return dispatch_qpk<D, 16, PG>(qpk, a, plan, s);
        case 32: return dispatch_qpk<D, 32, PG>(qpk, a, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const loopvq_cache &cc, const DecodePlan &plan, int layer, int t,
                          const uint16_t *q, const int32_t *starts, int start_all, const int32_t *lens, int max_len,
                          float scale, float *out, float *lse, void *workspace, cudaStream_t s,
                          const loopvq_tasq *tq) {
    DecodeArgs a{};
    const int beta = t / cc.Tc;
    a.idx = cc.idx + idx_base(cc, layer, beta, 0, 0);
    a.slk = cc.slices + slice_base(cc, layer, t, 0, 0);
    a.slv = cc.slices + slice_base(cc, layer, t, 1, 0);
    a.rope = cc.rope;
    a.q = q;
    a.lens = lens;
    a.starts = starts;
    a.start_all = start_all;
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
    if (tq) {
        const int NB = cc.T / cc.Tc;
        a.tw = tq->w + ((size_t)layer * cc.T + t) * cc.Hkv * cc.D;
        a.tperm = tq->perm + ((size_t)layer * NB + beta) * cc.Hkv * (cc.D / 2);
        a.tsig = tq->sigma + ((size_t)layer * cc.T + t) * cc.B * cc.Nmax;
        if (ncb_of(cc) != 1) return cudaErrorInvalidValue;
        if (cc.D == 128 && cc.c == 4) return dispatch_tq_qpk<128, 4>(qpk, a, plan, s);
        if (cc.D == 128 && cc.c == 8) return dispatch_tq_qpk<128, 8>(qpk, a, plan, s);
        if (cc.D == 64 && cc.c == 4) return dispatch_tq_qpk<64, 4>(qpk, a, plan, s);
        if (cc.D == 64 && cc.c == 8) return dispatch_tq_qpk<64, 8>(qpk, a, plan, s);
        return cudaErrorInvalidValue;
    }
    const bool pg = ncb_of(cc) > 1;
    if (cc.D == 128) return pg ? dispatch_c<128, true>(cc.c, qpk, a, plan, s) : dispatch_c<128, false>(cc.c, qpk, a, plan, s);
    if (cc.D == 64) return pg ? dispatch_c<64, true>(cc.c, qpk, a, plan, s) : dispatch_c<64, false>(cc.c, qpk, a, plan, s);
    return cudaErrorInvalidValue;
}

}  // namespace loopvq
