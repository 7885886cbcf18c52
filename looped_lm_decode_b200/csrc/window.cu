// The bf16 window of the coded cache and its decode-time life cycle.
//
// LoopVQ paper, Sec. 4.3 "Cache layout": the first n_s (sink) and the most recent n_r tokens of a
// request stay in bf16 in pages of 8 tokens, all other tokens are coded; "Encoding": during
// decode the oldest recent page is encoded once the window holds a page more than n_r;
// "Attention": one kernel attends to the bf16 tokens, another to the coded ones, and the results
// are combined through their log-sum-exps.
//
// Per (layer, loop step, sequence, KV head) the window has W = n_s + n_r + 8 slots: the sink, then
// the recent tokens oldest first.  Keys are kept rotated (for attention) and before RoPE (for the
// encoder).  The per-sequence counters fill (slots in use) and coded_end (end of the coded tokens)
// live on the device, so a decode step never waits for the host:
//   advance: full windows whose coded cache has room for a page encode their oldest page into it
//            (every layer and block, one launch), move the recent slots down by 8 (one launch) and
//            update the counters; then every sequence reserves the new token's slot.  A full window
//            without room does not roll and sets the fault word (LOOPVQ_ERR_OVERFLOW).
//   append:  the new token's K (rotated and not) and V of one (layer, loop step) go to slot fill-1.
//   attend:  the coded kernel over [n_s, coded_end), whose merge kernel also attends to the window
//            slots and combines both parts through their log-sum-exps (two launches in all).
#include "encode_common.cuh"

namespace loopvq {

struct WinEncArgs {
    const uint16_t *k_pre, *v;   // window base; element (l, t, b, h, slot, d)
    uint32_t *idx;               // coded cache words of layer 0, block 0, b = 0, h = 0
    const uint16_t *cb;          // codebook of layer 0, block 0, kv = 0, h = 0
    const int32_t *fill, *coded_end;
    int L, T, NB, B, Hkv, K, Nmax, W, n_sink;
};

// A sequence rolls when its window is full and the coded cache has room for the page; the three
// kernels of an advance all take this decision from the same counters.
__device__ __forceinline__ bool rolls(const int32_t *fill, const int32_t *coded_end, int b, int W, int Nmax) {
    return __ldg(fill + b) >= W && __ldg(coded_end + b) + 8 <= Nmax;
}

// One thread per index word of the oldest recent page: token i < 8 of the page, pair-group p.
// Grid: (ceil(8 NP / 128), L * NB * Hkv, B); the CTA's (layer, block, head) share a codebook.
template <int D, int C, int TC>
__global__ void __launch_bounds__(128) window_page_encode_kernel(const WinEncArgs a) {
    constexpr int G = C * TC;
    constexpr int NP = D / (2 * C);
    extern __shared__ __align__(16) float ecb[];             // [2][K][G] fp32
    const int b = blockIdx.z;
    if (!rolls(a.fill, a.coded_end, b, a.W, a.Nmax)) return; // uniform per CTA
    const int h = blockIdx.y % a.Hkv;
    const int lb = blockIdx.y / a.Hkv;
    const int block = lb % a.NB, layer = lb / a.NB;
    const int K = a.K;
    stage_codebooks<G>(ecb, a.cb + (size_t)(layer * a.NB + block) * 2 * a.Hkv * K * G, a.Hkv, h, K);
    __syncthreads();

    const int wl = blockIdx.x * blockDim.x + threadIdx.x;
    if (wl >= 8 * NP) return;
    const int i = wl / NP, p = wl % NP;
    const int n = __ldg(a.coded_end + b) + i;                // token position of the word (< Nmax: it rolls)
    const int slot = a.n_sink + i;
    const size_t tstride = (size_t)a.B * a.Hkv * a.W * D;    // one loop step of the window
    float z[4][G];
#pragma unroll
    for (int m = 0; m < TC; ++m) {
        const size_t row = ((size_t)(layer * a.T + block * TC + m) * tstride) +
                           (((size_t)b * a.Hkv + h) * a.W + slot) * D;
#pragma unroll
        for (int ii = 0; ii < C; ++ii) {
            z[0][ii * TC + m] = bf16_to_f32(__ldg(a.k_pre + row + p * C + ii));
            z[1][ii * TC + m] = bf16_to_f32(__ldg(a.k_pre + row + (p + NP) * C + ii));
            z[2][ii * TC + m] = bf16_to_f32(__ldg(a.v + row + p * C + ii));
            z[3][ii * TC + m] = bf16_to_f32(__ldg(a.v + row + (p + NP) * C + ii));
        }
    }
    const uint32_t word = nearest_word<G>(z, ecb, ecb + (size_t)K * G, K);
    const size_t per_bh = idx_words_per_bh(a.Nmax, D, C);
    a.idx[((size_t)(layer * a.NB + block) * a.B * a.Hkv + (size_t)b * a.Hkv + h) * per_bh + idx_word(n, p, NP)] =
        word;
}

// Move recent slots n_sink+8 .. W-1 down to n_sink .. W-9 in k_rot, k_pre and v of full windows.
// Grid: (L * T * Hkv, B); the rows are staged whole in shared memory, so the overlapping copy
// reads every slot before any is written.
__global__ void __launch_bounds__(256) window_shift_kernel(uint16_t *k_rot, uint16_t *k_pre, uint16_t *v,
                                                           const int32_t *fill, const int32_t *coded_end, int B,
                                                           int Hkv, int D, int W, int n_sink, int n_recent,
                                                           int Nmax) {
    extern __shared__ __align__(16) uint4 stage[];
    const int b = blockIdx.y;
    if (!rolls(fill, coded_end, b, W, Nmax)) return;
    const int lt = blockIdx.x / Hkv, h = blockIdx.x % Hkv;
    const size_t row = (((size_t)lt * B + b) * Hkv + h) * (size_t)W * D;
    const int n16 = n_recent * D / 8;                        // 16-byte words moved
    uint16_t *bufs[3] = {k_rot, k_pre, v};
    for (int k = 0; k < 3; ++k) {
        uint4 *dst = reinterpret_cast<uint4 *>(bufs[k] + row + (size_t)n_sink * D);
        const uint4 *src = reinterpret_cast<const uint4 *>(bufs[k] + row + (size_t)(n_sink + 8) * D);
        for (int i = threadIdx.x; i < n16; i += blockDim.x) stage[i] = src[i];
        __syncthreads();
        for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = stage[i];
        __syncthreads();
    }
}

// A full window whose coded cache has no room for the page does not roll: its counters stay, and the
// fault word records it (loopvq_fault_check reports LOOPVQ_ERR_OVERFLOW).
__global__ void window_counters_kernel(int32_t *fill, int32_t *coded_end, int B, int W, int Nmax,
                                       unsigned int *fault) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    int f = fill[b];
    if (f >= W) {
        if (coded_end[b] + 8 > Nmax) {
            atomicOr(fault, kFaultWindowFull);
            return;
        }
        f -= 8;
        coded_end[b] += 8;
    }
    fill[b] = f + 1;                                         // the new token's slot
}

// Slot fill_b - 1 of every (b, h) receives the token's rotated key, key before RoPE and value.
__global__ void window_append_kernel(uint16_t *k_rot, uint16_t *k_pre, uint16_t *v, const uint16_t *nk_rot,
                                     const uint16_t *nk_pre, const uint16_t *nv, const int32_t *fill, int B,
                                     int Hkv, int D, int W, size_t lt_off) {
    const int b = blockIdx.x, h = blockIdx.y;
    const int slot = __ldg(fill + b) - 1;
    if (slot < 0 || slot >= W) return;
    const size_t dst = lt_off + (((size_t)b * Hkv + h) * W + slot) * D;
    const size_t src = ((size_t)b * Hkv + h) * D;
    for (int i = threadIdx.x; i < D / 8; i += blockDim.x) {
        reinterpret_cast<uint4 *>(k_rot + dst)[i] = reinterpret_cast<const uint4 *>(nk_rot + src)[i];
        reinterpret_cast<uint4 *>(k_pre + dst)[i] = reinterpret_cast<const uint4 *>(nk_pre + src)[i];
        reinterpret_cast<uint4 *>(v + dst)[i] = reinterpret_cast<const uint4 *>(nv + src)[i];
    }
}

// ------------------------------------------------------------------ host side

int window_slots(const loopvq_window &w) { return w.n_sink + w.n_recent + 8; }

template <int D, int C, int TC>
static cudaError_t launch_page_encode(const WinEncArgs &a, cudaStream_t s) {
    constexpr int NP = D / (2 * C);
    const size_t smem = 2 * (size_t)a.K * C * TC * sizeof(float);
    auto k = window_page_encode_kernel<D, C, TC>;
    cudaError_t e = ensure_dynamic_smem((const void *)k, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((8 * NP + 127) / 128, a.L * a.NB * a.Hkv, a.B);
    k<<<grid, 128, smem, s>>>(a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_page_encode(int c, int tc, const WinEncArgs &a, cudaStream_t s) {
    if (c == 4 && tc == 4) return launch_page_encode<D, 4, 4>(a, s);
    if (c == 4 && tc == 2) return launch_page_encode<D, 4, 2>(a, s);
    if (c == 4 && tc == 1) return launch_page_encode<D, 4, 1>(a, s);
    if (c == 8 && tc == 4) return launch_page_encode<D, 8, 4>(a, s);
    if (c == 8 && tc == 2) return launch_page_encode<D, 8, 2>(a, s);
    if (c == 8 && tc == 1) return launch_page_encode<D, 8, 1>(a, s);
    if (c == 16 && tc == 2) return launch_page_encode<D, 16, 2>(a, s);
    if (c == 16 && tc == 1) return launch_page_encode<D, 16, 1>(a, s);
    if (c == 32 && tc == 1) return launch_page_encode<D, 32, 1>(a, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_window_advance(const loopvq_window &w, const loopvq_cache &cc, cudaStream_t s) {
    const int W = window_slots(w);
    WinEncArgs a{};
    a.k_pre = w.k_pre;
    a.v = w.v;
    a.idx = cc.idx;
    a.cb = cc.codebook;
    a.fill = w.fill;
    a.coded_end = w.coded_end;
    a.L = cc.L;
    a.T = cc.T;
    a.NB = cc.T / cc.Tc;
    a.B = cc.B;
    a.Hkv = cc.Hkv;
    a.K = cc.K;
    a.Nmax = cc.Nmax;
    a.W = W;
    a.n_sink = w.n_sink;
    cudaError_t e = cc.D == 128 ? dispatch_page_encode<128>(cc.c, cc.Tc, a, s)
                                : dispatch_page_encode<64>(cc.c, cc.Tc, a, s);
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)w.n_recent * w.D * 2;
    e = ensure_dynamic_smem((const void *)window_shift_kernel, smem);
    if (e != cudaSuccess) return e;
    unsigned int *fault = nullptr;
    if ((e = fault_word_for_current_device(&fault)) != cudaSuccess) return e;
    window_shift_kernel<<<dim3(w.L * w.T * w.Hkv, w.B), 256, smem, s>>>(w.k_rot, w.k_pre, w.v, w.fill, w.coded_end,
                                                                         w.B, w.Hkv, w.D, W, w.n_sink, w.n_recent,
                                                                         cc.Nmax);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    window_counters_kernel<<<(w.B + 127) / 128, 128, 0, s>>>(w.fill, w.coded_end, w.B, W, cc.Nmax, fault);
    return cudaGetLastError();
}

cudaError_t launch_window_append(const loopvq_window &w, int layer, int t, const uint16_t *k_rot,
                                 const uint16_t *k_pre, const uint16_t *v, cudaStream_t s) {
    const int W = window_slots(w);
    const size_t lt_off = ((size_t)layer * w.T + t) * w.B * w.Hkv * W * w.D;
    window_append_kernel<<<dim3(w.B, w.Hkv), 32, 0, s>>>(w.k_rot, w.k_pre, w.v, k_rot, k_pre, v, w.fill, w.B,
                                                         w.Hkv, w.D, W, lt_off);
    return cudaGetLastError();
}

// Workspace: the coded kernel's partial records.

size_t window_ws_bytes(const loopvq_window &w, const loopvq_cache &cc, int max_coded) {
    (void)w;
    return plan_decode(cc, max_coded).ws_bytes;
}

// The coded kernel over tokens [n_sink, coded_end_b); its merge kernel attends to the window slots
// [0, fill_b) of (layer, t) itself and folds them into the log-sum-exp merge (decode_merge.cuh).  With
// k_rot, k_pre, v given, slot fill_b - 1 is the token they hold, which the merge kernel also writes into
// the window (the work of launch_window_append, without its launch).
cudaError_t launch_window_decode(const loopvq_window &w, const loopvq_cache &cc, int layer, int t, const uint16_t *q,
                                 int max_coded, float scale, float *out, float *lse, void *ws, cudaStream_t s,
                                 const uint16_t *k_rot, const uint16_t *k_pre, const uint16_t *v) {
    const int W = window_slots(w);
    const size_t off = ((size_t)layer * w.T + t) * w.B * w.Hkv * W * w.D;
    const DecodePlan pc = plan_decode(cc, max_coded);
    const WindowAppend app{k_rot, k_pre, v, w.k_rot + off, w.k_pre + off, w.v + off};
    return launch_decode(cc, pc, layer, t, q, nullptr, w.n_sink, w.coded_end, max_coded, scale, out, lse, ws, s,
                         nullptr, w.k_rot + off, w.v + off, w.fill, W, k_rot != nullptr ? &app : nullptr);
}

}  // namespace loopvq
