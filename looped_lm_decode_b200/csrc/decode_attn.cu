// Decode attention over the loop-axis coded cache, one loop step of one layer:
// launch planning and dispatch.  The kernels are in decode_split.cuh, decode_mha.cuh, decode_gqa.cuh and
// decode_merge.cuh, on the shared tile space of decode_kernel.cuh.
//
// LoopVQ paper, Sec. 4.3 "Attention": the quantized tokens are divided into
// splits processed by separate thread blocks, and the partial outputs of all
// splits are combined using the log-sum-exp of their scores.
#include <math.h>

#include "decode_kernel.cuh"
#include "decode_merge.cuh"
#include "decode_split.cuh"
#include "decode_gqa.cuh"
#include "decode_mha.cuh"

namespace loopvq {

// ------------------------------------------------------------------ host side
//
// Exactly one wave of resident CTAs shares the tile space evenly (decode_kernel.cuh): with a shared
// codebook, two CTAs of 8 warps per SM (64 KiB of slice replicas plus a 2-deep prefetch queue each;
// the shared memory left over serves as L1 for the RoPE rows); with one codebook per channel group,
// one CTA of 16 warps per SM (128 KiB of tables).  Measured at ctx32k: a second wave, or three CTAs
// per SM at 80 registers, is 3 to 10 % slower.  decode_mha_kernel runs two CTAs of 8 warps per SM
// (2-deep index ring per warp): one CTA of 16 warps is 3% slower at ctx32k and 8% at ctx4k, a 3-deep
// ring 1% slower.

static constexpr int kSms = 148;                           // B200; more CTAs than fit only add a wave
static constexpr int kWords = 1;                           // index words per lane per iteration (4-token tiles)
static constexpr long kMinTiles = 128;                     // tiles per CTA below which fewer CTAs are used

struct KernelShape {
    int warps, min_blocks, depth;
};
static constexpr KernelShape kernel_shape(bool pg, int qpk) {
    return pg ? KernelShape{16, 1, 4} : KernelShape{8, 2, 2};
}

// Tables, the per-thread index queue and, with at most 2 query heads per KV head, the slot records
// (decode_split_kernel keeps its tables across the pieces of one KV head then).
static size_t ring_smem_bytes(bool pg, int qpk, int D) {
    const KernelShape k = kernel_shape(pg, qpk);
    const size_t nslot = (size_t)k.warps * (32 / (D / 8));
    const size_t recs = qpk <= 2 ? nslot * qpk * (D + 4) * sizeof(float) : 0;
    return (pg ? 131072 : 65536) + (size_t)k.depth * k.warps * 32 * 16 * kWords + recs;
}

// decode_mha_kernel (one query head per KV head, D = 128, groups of 4 channels or of 16, one shared
// codebook)
// runs the step-4 RoPE recurrence in plain form on the frequencies f < D/4 and in difference form on
// f >= D/4; it needs |sin 4w_f| >= 0.04 on the first (the recurrence's rounding grows as 1/|sin 4w|),
// 4w_f <= 1 on the second, and table rows 2 and 4.  With the base 1e4: min |sin 4w| = 0.046 (f = 31).
static constexpr int kMhaWarps = 8, kMhaMinBlocks = 2, kMhaDepth = 2;

static bool mha_applies(const loopvq_cache &cc) {
    if (cc.D != 128 || (cc.c != 4 && cc.c != 16) || cc.Hq != cc.Hkv || ncb_of(cc) != 1 || cc.Nmax < 8) return false;
    for (int f = 0; f < 64; ++f) {
        const double w = pow((double)cc.theta, -2.0 * f / 128.0);
        if (f < 32 ? fabs(sin(4.0 * w)) < 0.04 : 4.0 * w > 1.0) return false;
    }
    return true;
}

template <int D>
static cudaError_t launch_merge(const DecodeArgs &a, cudaStream_t s);

// decode_gqa_kernel (4 query heads per KV head, D = 128, groups of 8 channels, one shared codebook):
// one CTA of 8 warps per SM (254 registers per thread, 152.5 KiB of shared memory), 2-stage index ring
// per warp.
static constexpr int kGqaWarps = 8, kGqaMinBlocks = 1, kGqaDepth = 2;

static bool gqa_applies(const loopvq_cache &cc) {
    return cc.D == 128 && cc.c == 8 && cc.Hq == 4 * cc.Hkv && ncb_of(cc) == 1 && cc.Nmax >= 8;
}

static cudaError_t launch_gqa(const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    using S = GqaSmem<kGqaWarps, kGqaDepth>;
    auto kern = decode_gqa_kernel<kGqaWarps, kGqaMinBlocks, kGqaDepth>;
    cudaError_t e = ensure_dynamic_smem((const void *)kern, S::kBytes);
    if (e != cudaSuccess) return e;
    if (plan.ncta > 0) {
        kern<<<plan.ncta, kGqaWarps * 32, S::kBytes, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_merge<128>(a, s);
}

template <bool TQ, int C>
static cudaError_t launch_mha(const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    using S = MhaSmem<kMhaWarps, kMhaDepth, 64u * (128 / (2 * C))>;
    auto kern = decode_mha_kernel<kMhaWarps, kMhaMinBlocks, kMhaDepth, TQ, C>;
    cudaError_t e = ensure_dynamic_smem((const void *)kern, S::kBytes);
    if (e != cudaSuccess) return e;
    if (plan.ncta > 0) {
        kern<<<plan.ncta, kMhaWarps * 32, S::kBytes, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_merge<128>(a, s);
}

DecodePlan plan_decode(const loopvq_cache &cc, int max_len, bool tasq) {
    DecodePlan p{};
    const bool pg = ncb_of(cc) > 1;
    const int qpk = cc.Hq / cc.Hkv;
    const KernelShape k = kernel_shape(pg, qpk);
    p.nbt = 1;
    p.nchunk = cc.B;
    p.mha = mha_applies(cc);                               // plain or TaSQ keys
    p.gqa = !tasq && gqa_applies(cc);
    // an upper bound of the tiles: every sequence at max_len
    const long tiles = (long)cc.B * cc.Hkv * ((max_len + 3) / 4);
    const long g = (tiles + kMinTiles - 1) / kMinTiles;
    const long cap = (long)kSms * (p.mha ? kMhaMinBlocks : p.gqa ? kGqaMinBlocks : k.min_blocks);
    p.ncta = max_len > 0 ? (int)(g < cap ? g : cap) : 0;
    p.npiece = cc.B * cc.Hkv + p.ncta;
    p.split_len = 0;
    p.nsplit = p.ncta;
    // the workspace covers either kernel's records, so one size serves plain and TaSQ calls
    const long cap_ws = (long)kSms * (k.min_blocks > kMhaMinBlocks ? k.min_blocks : kMhaMinBlocks);
    const long npiece_ws = (long)cc.B * cc.Hkv + (max_len > 0 ? (g < cap_ws ? g : cap_ws) : 0);
    const size_t o_bytes = (size_t)npiece_ws * qpk * cc.D * sizeof(float);
    const size_t ml_bytes = (size_t)npiece_ws * qpk * sizeof(float2);
    p.ws_bytes = ((o_bytes + 255) & ~(size_t)255) + ml_bytes;
    return p;
}

template <int D, int C, int QPK, bool PG, bool TQ = false>
static cudaError_t launch_t(const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s) {
    constexpr KernelShape K = kernel_shape(PG, QPK);
    constexpr int NSLOT = K.warps * (32 / (D / 8));
    const size_t red = (size_t)NSLOT * QPK * (D + 4) * sizeof(float);
    const size_t smem = ring_smem_bytes(PG, QPK, D);
    if (red > smem) return cudaErrorInvalidConfiguration;   // the slot records fit (own area or the tables)
    // TaSQ with one query head per KV head carries the rotated query from tile to tile (XR): its
    // table values sit at permuted columns, 8 scalar loads per tile.  The plain kernels load the
    // table row one iteration ahead, which measured faster for them (143 vs 150 us at ctx32k).
    constexpr bool XR = TQ && QPK == 1;
    auto kern = decode_split_kernel<D, C, QPK, K.warps, K.min_blocks, K.depth, kWords, PG, TQ, XR>;
    cudaError_t e = ensure_dynamic_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    if (plan.ncta > 0) {
        kern<<<plan.ncta, K.warps * 32, smem, s>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_merge<D>(a, s);
}

// the merge as a programmatic dependent launch: it overlaps the split kernel's last CTAs
template <int D>
static cudaError_t launch_merge(const DecodeArgs &a, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.Hq);
    cfg.blockDim = dim3(D);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, merge_kernel<D>, a);
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
                          const loopvq_tasq *tq, const uint16_t *wk, const uint16_t *wv, const int32_t *wfill,
                          int W, const WindowAppend *app) {
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
    const size_t o_bytes = (size_t)plan.npiece * (cc.Hq / cc.Hkv) * cc.D * sizeof(float);
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
    a.ncta = plan.ncta;
    a.qscale = scale * 1.44269504088896340736f;
    a.wk = wk;
    a.wv = wv;
    a.wfill = wfill;
    a.W = W;
    if (app != nullptr) {
        a.nk = app->k_rot;
        a.nkp = app->k_pre;
        a.nv = app->v;
        a.wk_w = app->w_k_rot;
        a.wkp_w = app->w_k_pre;
        a.wv_w = app->w_v;
    }
    const int qpk = cc.Hq / cc.Hkv;
    if (tq) {
        const int NB = cc.T / cc.Tc;
        a.tw = tq->w + ((size_t)layer * cc.T + t) * cc.Hkv * cc.D;
        a.tperm = tq->perm + ((size_t)layer * NB + beta) * cc.Hkv * (cc.D / 2);
        a.tsig = tq->sigma + ((size_t)layer * cc.T + t) * cc.B * cc.Nmax;
        if (ncb_of(cc) != 1) return cudaErrorInvalidValue;
        if (plan.mha && cc.c == 4) return launch_mha<true, 4>(a, plan, s);
        if (cc.D == 128 && cc.c == 4) return dispatch_tq_qpk<128, 4>(qpk, a, plan, s);
        if (cc.D == 128 && cc.c == 8) return dispatch_tq_qpk<128, 8>(qpk, a, plan, s);
        if (cc.D == 64 && cc.c == 4) return dispatch_tq_qpk<64, 4>(qpk, a, plan, s);
        if (cc.D == 64 && cc.c == 8) return dispatch_tq_qpk<64, 8>(qpk, a, plan, s);
        return cudaErrorInvalidValue;
    }
    const bool pg = ncb_of(cc) > 1;
    if (plan.mha) return cc.c == 4 ? launch_mha<false, 4>(a, plan, s) : launch_mha<false, 16>(a, plan, s);
    if (plan.gqa) return launch_gqa(a, plan, s);
    if (cc.D == 128) return pg ? dispatch_c<128, true>(cc.c, qpk, a, plan, s) : dispatch_c<128, false>(cc.c, qpk, a, plan, s);
    if (cc.D == 64) return pg ? dispatch_c<64, true>(cc.c, qpk, a, plan, s) : dispatch_c<64, false>(cc.c, qpk, a, plan, s);
    return cudaErrorInvalidValue;
}

}  // namespace loopvq
