// Internal declarations shared by the CUDA translation units of libloopvq.
// Layout arithmetic for the buffers described in include/loopvq.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/loopvq.h"

namespace loopvq {

// Offsets (in elements) of the first element of a sub-array.
__host__ __device__ inline size_t idx_words_per_bh(int Nmax, int D, int c) {
    return (size_t)Nmax * (size_t)(D / (2 * c));
}
// idx base of (layer, block, b, h)
__host__ __device__ inline size_t idx_base(const loopvq_cache &cc, int layer, int block, int b, int h) {
    const int NB = cc.T / cc.Tc;
    return ((((size_t)layer * NB + block) * cc.B + b) * cc.Hkv + h) * idx_words_per_bh(cc.Nmax, cc.D, cc.c);
}
// word of token n, pair-group p within a (layer, block, b, h) run
__host__ __device__ inline size_t idx_word(int n, int p, int NP) {
    return (((size_t)(n >> 2) * NP + p) << 2) + (n & 3);
}
// slice base of (layer, t, kv, h): [K][c] bf16
// codebooks per (layer, block, head, K|V): 1 (shared) or D/c (one per channel group)
__host__ __device__ inline int ncb_of(const loopvq_cache &cc) { return cc.ncb > 1 ? cc.ncb : 1; }
__host__ __device__ inline size_t slice_base(const loopvq_cache &cc, int layer, int t, int kv, int h) {
    return ((((size_t)layer * cc.T + t) * 2 + kv) * cc.Hkv + h) * (size_t)cc.K * cc.c * ncb_of(cc);
}
// codebook base of (layer, block, kv, h): [NCB][K][G] bf16
__host__ __device__ inline size_t codebook_base(const loopvq_cache &cc, int layer, int block, int kv, int h) {
    const int NB = cc.T / cc.Tc;
    return ((((size_t)layer * NB + block) * 2 + kv) * cc.Hkv + h) * (size_t)cc.K * (cc.c * cc.Tc) * ncb_of(cc);
}

// bf16 bit pattern -> fp32 (exact)
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// Sets the thread-local message returned by loopvq_last_error().
void set_last_error(const char *msg);

// Bits of the per-GPU fault word (faults.cu), reported by loopvq_fault_check.
constexpr unsigned int kFaultEncodeWait = 1u;   // a tensor-core encode's bounded wait ran out
constexpr unsigned int kFaultWindowFull = 2u;   // a window roll found the coded cache full
// Device address of the fault word on the current device (looked up once per device).
cudaError_t fault_word_for_current_device(unsigned int **out);
// Bound on each wait of the tensor-core encoder for its own contraction (loopvq_set_wait_limit_ns).
unsigned long long wait_limit_ns();

// Raises a kernel's dynamic shared-memory limit on the current device to at least `bytes`.  The
// attribute is set on the first such request (or a larger one) per kernel and device only, so steady
// launches make no attribute call: less host time per call, and nothing but launches inside a CUDA
// graph capture.
cudaError_t ensure_dynamic_smem(const void *kern, size_t bytes);

// Launchers (host); each returns a cudaError_t from the launch.
cudaError_t launch_prepare(const loopvq_cache &cc, cudaStream_t s);
cudaError_t launch_encode(const loopvq_cache &cc, int layer, int block, const void *xk, const void *xv,
                          int x_dtype, const int64_t *strides, int b0, int nb, int tok0, int ntok,
                          cudaStream_t s);
cudaError_t launch_dequant(const loopvq_cache &cc, int layer, int t, int kv, int b, int tok0, int ntok,
                           int apply_rope, float *out, cudaStream_t s);

struct DecodePlan {
    int split_len;      // bf16 kernel: tokens per split (multiple of 4)
    int nsplit;         // bf16 kernel: splits covering max_len; coded kernel: its CTAs
    int ncta;           // coded kernel: CTAs sharing the tile space
    int npiece;         // coded kernel: partial records (segments + CTAs)
    int nbt;            // sequences per thread block
    int nchunk;         // ceil(B / nbt)
    bool mha;           // coded kernel: decode_mha_kernel applies (one query head per KV head, D 128, c 4)
    bool gqa;           // coded kernel: decode_gqa_kernel applies (4 query heads per KV head, D 128, c 8)
    size_t ws_bytes;    // workspace needed
};
DecodePlan plan_decode(const loopvq_cache &cc, int max_len, bool tasq = false);
// A window token appended by the windowed decode's merge kernel: its rows [B][Hkv][D] and the window
// arrays of (layer, t) it is written to.
struct WindowAppend {
    const uint16_t *k_rot, *k_pre, *v;
    uint16_t *w_k_rot, *w_k_pre, *w_v;
};
cudaError_t launch_decode(const loopvq_cache &cc, const DecodePlan &plan, int layer, int t,
                          const uint16_t *q, const int32_t *starts, int start_all, const int32_t *lens, int max_len,
                          float scale, float *out, float *lse, void *workspace, cudaStream_t s,
                          const loopvq_tasq *tq = nullptr, const uint16_t *wk = nullptr,
                          const uint16_t *wv = nullptr, const int32_t *wfill = nullptr, int W = 0,
                          const WindowAppend *app = nullptr);
cudaError_t launch_tasq_encode(const loopvq_cache &cc, const loopvq_tasq &tq, int layer, int block, const void *xk,
                               const void *xv, int x_dtype, const int64_t *strides, int b0, int nb, int tok0, int ntok,
                               cudaStream_t s);
cudaError_t launch_tasq_encode_tc(const loopvq_cache &cc, const loopvq_tasq &tq, int layer, int block, const void *xk,
                                  const void *xv, const int64_t *strides, int b0, int nb, int tok0, int ntok,
                                  cudaStream_t s);
DecodePlan plan_bf16(const loopvq_bf16_cache &c, int max_len);
cudaError_t launch_bf16_decode(const loopvq_bf16_cache &c, const DecodePlan &plan, const uint16_t *q,
                               const int32_t *starts, const int32_t *lens, int max_len, float scale, float *out,
                               float *lse, void *workspace, cudaStream_t s);
cudaError_t launch_merge2(const float *out_a, const float *lse_a, const float *out_b, const float *lse_b, int rows,
                          int D, float *out, float *lse, cudaStream_t s);
int window_slots(const loopvq_window &w);
cudaError_t launch_window_advance(const loopvq_window &w, const loopvq_cache &cc, cudaStream_t s);
cudaError_t launch_window_append(const loopvq_window &w, int layer, int t, const uint16_t *k_rot,
                                 const uint16_t *k_pre, const uint16_t *v, cudaStream_t s);
size_t window_ws_bytes(const loopvq_window &w, const loopvq_cache &cc, int max_coded);
cudaError_t launch_window_decode(const loopvq_window &w, const loopvq_cache &cc, int layer, int t, const uint16_t *q,
                                 int max_coded, float scale, float *out, float *lse, void *ws, cudaStream_t s,
                                 const uint16_t *k_rot = nullptr, const uint16_t *k_pre = nullptr,
                                 const uint16_t *v = nullptr);

}  // namespace loopvq
