// C ABI of libloopvq: host-side validation, then launches on the caller's stream.
// Every entry point checks its arguments before launching anything and never
// allocates or synchronises.
#include <cmath>
#include <map>
#include <mutex>
#include <utility>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "loopvq_internal.cuh"

namespace {

thread_local char g_err[512] = "";

// Opt-in shared memory per CTA on B200 (227 KiB).
constexpr size_t kMaxOptinSmem = 232448;

loopvq_status fail(loopvq_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

loopvq_status cuda_fail(cudaError_t e, const char *where) {
    return fail(LOOPVQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every call.
loopvq_status check_shape(const loopvq_cache *cc) {
    if (!cc) return fail(LOOPVQ_ERR_INVALID_ARG, "cache is NULL");
    if (cc->L <= 0 || cc->T <= 0 || cc->Tc <= 0 || cc->Hkv <= 0 || cc->Hq <= 0 || cc->D <= 0 || cc->c <= 0 ||
        cc->K <= 0 || cc->B <= 0 || cc->Nmax <= 0)
        return fail(LOOPVQ_ERR_INVALID_ARG, "all shape fields must be positive");
    if (cc->T % cc->Tc != 0) return fail(LOOPVQ_ERR_INVALID_ARG, "T=%d is not a multiple of Tc=%d", cc->T, cc->Tc);
    if (cc->Hq % cc->Hkv != 0) return fail(LOOPVQ_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", cc->Hq, cc->Hkv);
    if (cc->K > 256) return fail(LOOPVQ_ERR_INVALID_ARG, "K=%d exceeds 256 (8-bit codes)", cc->K);
    if (cc->Nmax % 4 != 0) return fail(LOOPVQ_ERR_INVALID_ARG, "Nmax=%d is not a multiple of 4", cc->Nmax);
    if (cc->D != 64 && cc->D != 128) return fail(LOOPVQ_ERR_UNSUPPORTED, "D=%d (supported: 64, 128)", cc->D);
    if (cc->c != 4 && cc->c != 8 && cc->c != 16 && cc->c != 32)
        return fail(LOOPVQ_ERR_UNSUPPORTED, "c=%d (supported: 4, 8, 16, 32)", cc->c);
    if (cc->Tc != 1 && cc->Tc != 2 && cc->Tc != 4) return fail(LOOPVQ_ERR_UNSUPPORTED, "Tc=%d (supported: 1, 2, 4)", cc->Tc);
    if (cc->c * cc->Tc > 32)
        return fail(LOOPVQ_ERR_UNSUPPORTED, "G = c*Tc = %d (supported: up to 32)", cc->c * cc->Tc);
    const int qpk = cc->Hq / cc->Hkv;
    if (qpk != 1 && qpk != 2 && qpk != 4 && qpk != 8)
        return fail(LOOPVQ_ERR_UNSUPPORTED, "Hq/Hkv=%d (supported: 1, 2, 4, 8)", qpk);
    if (!(cc->theta > 0.f) || !std::isfinite(cc->theta)) return fail(LOOPVQ_ERR_INVALID_ARG, "theta must be positive");
    if (cc->ncb != 0 && cc->ncb != 1 && cc->ncb != cc->D / cc->c)
        return fail(LOOPVQ_ERR_INVALID_ARG, "ncb=%d (1 shared, or D/c=%d per channel group)", cc->ncb, cc->D / cc->c);
    return LOOPVQ_OK;
}

loopvq_status check_ptr(const void *p, const char *name) {
    if (!p) return fail(LOOPVQ_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(p)) return fail(LOOPVQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return LOOPVQ_OK;
}

#define LQ_TRY(x)                              \
    do {                                       \
        loopvq_status _s = (x);                \
        if (_s != LOOPVQ_OK) return _s;        \
    } while (0)

}  // namespace

namespace loopvq {
void set_last_error(const char *msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

cudaError_t ensure_dynamic_smem(const void *kern, size_t bytes) {
    if (bytes <= 48u * 1024u) return cudaSuccess;          // within the default limit
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> done;
    std::lock_guard<std::mutex> lock(mu);
    size_t &cur = done[{kern, dev}];
    if (cur >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) cur = bytes;
    return e;
}
}  // namespace loopvq

extern "C" {

size_t loopvq_idx_words(const loopvq_cache *cc) {
    if (check_shape(cc) != LOOPVQ_OK) return 0;
    return (size_t)cc->L * (cc->T / cc->Tc) * cc->B * cc->Hkv * (size_t)cc->Nmax * (cc->D / (2 * cc->c));
}

size_t loopvq_codebook_elems(const loopvq_cache *cc) {
    if (check_shape(cc) != LOOPVQ_OK) return 0;
    return (size_t)cc->L * (cc->T / cc->Tc) * 2 * cc->Hkv * (size_t)cc->K * cc->c * cc->Tc * loopvq::ncb_of(*cc);
}

size_t loopvq_slice_elems(const loopvq_cache *cc) {
    if (check_shape(cc) != LOOPVQ_OK) return 0;
    return (size_t)cc->L * cc->T * 2 * cc->Hkv * (size_t)cc->K * cc->c * loopvq::ncb_of(*cc);
}

size_t loopvq_rope_elems(const loopvq_cache *cc) {
    if (check_shape(cc) != LOOPVQ_OK) return 0;
    return (size_t)cc->Nmax * cc->D;
}

loopvq_status loopvq_prepare(const loopvq_cache *cc, void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_shape(cc));
    LQ_TRY(check_ptr(cc->codebook, "codebook"));
    LQ_TRY(check_ptr(cc->slices, "slices"));
    LQ_TRY(check_ptr(cc->rope, "rope"));
    cudaError_t e = loopvq::launch_prepare(*cc, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_prepare");
    return LOOPVQ_OK;
}

loopvq_status loopvq_encode(const loopvq_cache *cc, int layer, int block, const void *xk, const void *xv,
                            int x_dtype, const int64_t x_strides[4], int b0, int nb, int tok0, int ntok,
                            void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_shape(cc));
    LQ_TRY(check_ptr(cc->idx, "idx"));
    LQ_TRY(check_ptr(cc->codebook, "codebook"));
    if (layer < 0 || layer >= cc->L) return fail(LOOPVQ_ERR_INVALID_ARG, "layer=%d out of [0, %d)", layer, cc->L);
    if (block < 0 || block >= cc->T / cc->Tc)
        return fail(LOOPVQ_ERR_INVALID_ARG, "block=%d out of [0, %d)", block, cc->T / cc->Tc);
    if (x_dtype != LOOPVQ_BF16 && x_dtype != LOOPVQ_FP32) return fail(LOOPVQ_ERR_INVALID_ARG, "x_dtype=%d", x_dtype);
    if (nb < 0 || ntok < 0 || b0 < 0 || tok0 < 0 || b0 + nb > cc->B || tok0 + ntok > cc->Nmax)
        return fail(LOOPVQ_ERR_INVALID_ARG, "sequence range [%d, %d) or token range [%d, %d) outside the cache",
                    b0, b0 + nb, tok0, tok0 + ntok);
    if (nb == 0 || ntok == 0) return LOOPVQ_OK;
    if (!xk || !xv) return fail(LOOPVQ_ERR_INVALID_ARG, "xk / xv is NULL");
    if (!x_strides) return fail(LOOPVQ_ERR_INVALID_ARG, "x_strides is NULL");
    for (int i = 0; i < 4; ++i)
        if (x_strides[i] < 0) return fail(LOOPVQ_ERR_INVALID_ARG, "negative stride %d", i);
    const size_t es = x_dtype == LOOPVQ_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(xk) | reinterpret_cast<uintptr_t>(xv)) % es)
        return fail(LOOPVQ_ERR_INVALID_ARG, "xk / xv not aligned to the element size");
    cudaError_t e = loopvq::launch_encode(*cc, layer, block, xk, xv, x_dtype, x_strides, b0, nb, tok0, ntok,
                                          (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_encode");
    return LOOPVQ_OK;
}

size_t loopvq_decode_workspace_bytes(const loopvq_cache *cc, int max_len) {
    if (check_shape(cc) != LOOPVQ_OK || max_len < 0 || max_len > cc->Nmax) return 0;
    return loopvq::plan_decode(*cc, max_len).ws_bytes;
}

static loopvq_status decode_common(const char *fn, const loopvq_cache *cc, int layer, int t, const uint16_t *q,
                                   const int32_t *starts, const int32_t *lens, int max_len, float scale, float *out,
                                   float *lse, void *workspace, size_t ws_bytes, void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_shape(cc));
    LQ_TRY(check_ptr(cc->idx, "idx"));
    LQ_TRY(check_ptr(cc->slices, "slices"));
    LQ_TRY(check_ptr(cc->rope, "rope"));
    LQ_TRY(check_ptr(q, "q"));
    LQ_TRY(check_ptr(lens, "lens"));
    LQ_TRY(check_ptr(out, "out"));
    if (starts && (reinterpret_cast<uintptr_t>(starts) & 3u))
        return fail(LOOPVQ_ERR_INVALID_ARG, "starts not 4-byte aligned");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(LOOPVQ_ERR_INVALID_ARG, "lse not 4-byte aligned");
    if (layer < 0 || layer >= cc->L) return fail(LOOPVQ_ERR_INVALID_ARG, "layer=%d out of [0, %d)", layer, cc->L);
    if (t < 0 || t >= cc->T) return fail(LOOPVQ_ERR_INVALID_ARG, "t=%d out of [0, %d)", t, cc->T);
    if (max_len < 0 || max_len > cc->Nmax)
        return fail(LOOPVQ_ERR_INVALID_ARG, "max_len=%d out of [0, Nmax=%d]", max_len, cc->Nmax);
    if (!std::isfinite(scale)) return fail(LOOPVQ_ERR_INVALID_ARG, "scale is not finite");
    if (scale <= 0.f) scale = 1.0f / std::sqrt((float)cc->D);
    const loopvq::DecodePlan plan = loopvq::plan_decode(*cc, max_len);
    if (plan.nsplit > 65535) return fail(LOOPVQ_ERR_UNSUPPORTED, "too many splits");
    if (!workspace || ws_bytes < plan.ws_bytes)
        return fail(LOOPVQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", plan.ws_bytes,
                    workspace ? ws_bytes : (size_t)0);
    if (!aligned16(workspace)) return fail(LOOPVQ_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    cudaError_t e = loopvq::launch_decode(*cc, plan, layer, t, q, starts, 0, lens, max_len, scale, out, lse,
                                          workspace, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return LOOPVQ_OK;
}

loopvq_status loopvq_decode_attn(const loopvq_cache *cc, int layer, int t, const uint16_t *q,
                                 const int32_t *lens, int max_len, float scale, float *out, float *lse,
                                 void *workspace, size_t ws_bytes, void *stream) {
    return decode_common("loopvq_decode_attn", cc, layer, t, q, nullptr, lens, max_len, scale, out, lse, workspace,
                         ws_bytes, stream);
}

loopvq_status loopvq_decode_attn_range(const loopvq_cache *cc, int layer, int t, const uint16_t *q,
                                       const int32_t *starts, const int32_t *lens, int max_len, float scale,
                                       float *out, float *lse, void *workspace, size_t ws_bytes, void *stream) {
    return decode_common("loopvq_decode_attn_range", cc, layer, t, q, starts, lens, max_len, scale, out, lse,
                         workspace, ws_bytes, stream);
}

static loopvq_status check_bf16(const loopvq_bf16_cache *c) {
    if (!c) return fail(LOOPVQ_ERR_INVALID_ARG, "cache is NULL");
    if (c->B <= 0 || c->Hkv <= 0 || c->Hq <= 0 || c->D <= 0 || c->Nmax <= 0)
        return fail(LOOPVQ_ERR_INVALID_ARG, "all shape fields must be positive");
    if (c->Hq % c->Hkv != 0) return fail(LOOPVQ_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", c->Hq, c->Hkv);
    if (c->D != 64 && c->D != 128) return fail(LOOPVQ_ERR_UNSUPPORTED, "D=%d (supported: 64, 128)", c->D);
    const int qpk = c->Hq / c->Hkv;
    if (qpk != 1 && qpk != 2 && qpk != 4 && qpk != 8)
        return fail(LOOPVQ_ERR_UNSUPPORTED, "Hq/Hkv=%d (supported: 1, 2, 4, 8)", qpk);
    LQ_TRY(check_ptr(c->k, "k"));
    LQ_TRY(check_ptr(c->v, "v"));
    return LOOPVQ_OK;
}

size_t loopvq_bf16_decode_workspace_bytes(const loopvq_bf16_cache *c, int max_len) {
    if (check_bf16(c) != LOOPVQ_OK || max_len < 0 || max_len > c->Nmax) return 0;
    return loopvq::plan_bf16(*c, max_len).ws_bytes;
}

loopvq_status loopvq_bf16_decode_attn(const loopvq_bf16_cache *c, const uint16_t *q, const int32_t *starts,
                                      const int32_t *lens, int max_len, float scale, float *out, float *lse,
                                      void *workspace, size_t ws_bytes, void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_bf16(c));
    LQ_TRY(check_ptr(q, "q"));
    LQ_TRY(check_ptr(lens, "lens"));
    LQ_TRY(check_ptr(out, "out"));
    if (starts && (reinterpret_cast<uintptr_t>(starts) & 3u))
        return fail(LOOPVQ_ERR_INVALID_ARG, "starts not 4-byte aligned");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(LOOPVQ_ERR_INVALID_ARG, "lse not 4-byte aligned");
    if (max_len < 0 || max_len > c->Nmax)
        return fail(LOOPVQ_ERR_INVALID_ARG, "max_len=%d out of [0, Nmax=%d]", max_len, c->Nmax);
    if (!std::isfinite(scale)) return fail(LOOPVQ_ERR_INVALID_ARG, "scale is not finite");
    if (scale <= 0.f) scale = 1.0f / std::sqrt((float)c->D);
    const loopvq::DecodePlan plan = loopvq::plan_bf16(*c, max_len);
    if (plan.nsplit > 65535) return fail(LOOPVQ_ERR_UNSUPPORTED, "too many splits");
    if (!workspace || ws_bytes < plan.ws_bytes)
        return fail(LOOPVQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", plan.ws_bytes,
                    workspace ? ws_bytes : (size_t)0);
    if (!aligned16(workspace)) return fail(LOOPVQ_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    cudaError_t e = loopvq::launch_bf16_decode(*c, plan, q, starts, lens, max_len, scale, out, lse, workspace,
                                               (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_bf16_decode_attn");
    return LOOPVQ_OK;
}

loopvq_status loopvq_merge2(const float *out_a, const float *lse_a, const float *out_b, const float *lse_b,
                            int rows, int D, float *out, float *lse, void *stream) {
    g_err[0] = 0;
    if (rows < 0) return fail(LOOPVQ_ERR_INVALID_ARG, "rows=%d is negative", rows);
    if (D != 64 && D != 128) return fail(LOOPVQ_ERR_UNSUPPORTED, "D=%d (supported: 64, 128)", D);
    if (rows == 0) return LOOPVQ_OK;
    if (!out_a || !lse_a || !out_b || !lse_b || !out) return fail(LOOPVQ_ERR_INVALID_ARG, "NULL input or output");
    const void *ptrs[6] = {out_a, lse_a, out_b, lse_b, out, lse};
    for (const void *p : ptrs)
        if (p && (reinterpret_cast<uintptr_t>(p) & 3u)) return fail(LOOPVQ_ERR_INVALID_ARG, "pointer not 4-byte aligned");
    cudaError_t e = loopvq::launch_merge2(out_a, lse_a, out_b, lse_b, rows, D, out, lse, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_merge2");
    return LOOPVQ_OK;
}

static loopvq_status check_tasq(const loopvq_cache *cc, const loopvq_tasq *tq) {
    LQ_TRY(check_shape(cc));
    if (loopvq::ncb_of(*cc) != 1) return fail(LOOPVQ_ERR_UNSUPPORTED, "TaSQ needs shared codebooks (ncb = 1)");
    if (cc->c != 4 && cc->c != 8) return fail(LOOPVQ_ERR_UNSUPPORTED, "TaSQ supports c = 4 or 8, not %d", cc->c);
    if (!tq) return fail(LOOPVQ_ERR_INVALID_ARG, "tasq is NULL");
    if (!tq->w || !tq->perm || !tq->sigma) return fail(LOOPVQ_ERR_INVALID_ARG, "tasq w, perm or sigma is NULL");
    if ((reinterpret_cast<uintptr_t>(tq->w) & 3u) || (reinterpret_cast<uintptr_t>(tq->perm) & 1u) ||
        (reinterpret_cast<uintptr_t>(tq->sigma) & 1u))
        return fail(LOOPVQ_ERR_INVALID_ARG, "tasq buffers misaligned");
    return LOOPVQ_OK;
}

size_t loopvq_tasq_w_elems(const loopvq_cache *cc) {
    if (check_shape(cc) != LOOPVQ_OK || loopvq::ncb_of(*cc) != 1 || (cc->c != 4 && cc->c != 8)) return 0;
    return (size_t)cc->L * cc->T * cc->Hkv * cc->D;
}

size_t loopvq_tasq_perm_elems(const loopvq_cache *cc) {
    if (check_shape(cc) != LOOPVQ_OK || loopvq::ncb_of(*cc) != 1 || (cc->c != 4 && cc->c != 8)) return 0;
    return (size_t)cc->L * (cc->T / cc->Tc) * cc->Hkv * (cc->D / 2);
}

size_t loopvq_tasq_sigma_elems(const loopvq_cache *cc) {
    if (check_shape(cc) != LOOPVQ_OK || loopvq::ncb_of(*cc) != 1 || (cc->c != 4 && cc->c != 8)) return 0;
    return (size_t)cc->L * cc->T * cc->B * (size_t)cc->Nmax;
}

loopvq_status loopvq_tasq_encode(const loopvq_cache *cc, const loopvq_tasq *tq, int layer, int block, const void *xk,
                                 const void *xv, int x_dtype, const int64_t x_strides[4], int b0, int nb, int tok0,
                                 int ntok, void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_tasq(cc, tq));
    LQ_TRY(check_ptr(cc->idx, "idx"));
    LQ_TRY(check_ptr(cc->codebook, "codebook"));
    if (!xk || !xv || !x_strides) return fail(LOOPVQ_ERR_INVALID_ARG, "xk, xv or x_strides is NULL");
    if (x_dtype != LOOPVQ_BF16 && x_dtype != LOOPVQ_FP32) return fail(LOOPVQ_ERR_INVALID_ARG, "x_dtype=%d", x_dtype);
    if (layer < 0 || layer >= cc->L) return fail(LOOPVQ_ERR_INVALID_ARG, "layer=%d out of [0, %d)", layer, cc->L);
    const int NB = cc->T / cc->Tc;
    if (block < 0 || block >= NB) return fail(LOOPVQ_ERR_INVALID_ARG, "block=%d out of [0, %d)", block, NB);
    if (b0 < 0 || nb < 0 || b0 + nb > cc->B) return fail(LOOPVQ_ERR_INVALID_ARG, "sequences [%d, %d) outside [0, %d)", b0, b0 + nb, cc->B);
    if (tok0 < 0 || ntok < 0 || tok0 + ntok > cc->Nmax)
        return fail(LOOPVQ_ERR_INVALID_ARG, "tokens [%d, %d) outside [0, %d)", tok0, tok0 + ntok, cc->Nmax);
    cudaError_t e = loopvq::launch_tasq_encode(*cc, *tq, layer, block, xk, xv, x_dtype, x_strides, b0, nb, tok0, ntok,
                                               (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_tasq_encode");
    return LOOPVQ_OK;
}

loopvq_status loopvq_tasq_decode_attn(const loopvq_cache *cc, const loopvq_tasq *tq, int layer, int t,
                                      const uint16_t *q, const int32_t *lens, int max_len, float scale, float *out,
                                      float *lse, void *workspace, size_t ws_bytes, void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_tasq(cc, tq));
    LQ_TRY(check_ptr(cc->idx, "idx"));
    LQ_TRY(check_ptr(cc->slices, "slices"));
    LQ_TRY(check_ptr(cc->rope, "rope"));
    LQ_TRY(check_ptr(q, "q"));
    LQ_TRY(check_ptr(lens, "lens"));
    LQ_TRY(check_ptr(out, "out"));
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(LOOPVQ_ERR_INVALID_ARG, "lse not 4-byte aligned");
    if (layer < 0 || layer >= cc->L) return fail(LOOPVQ_ERR_INVALID_ARG, "layer=%d out of [0, %d)", layer, cc->L);
    if (t < 0 || t >= cc->T) return fail(LOOPVQ_ERR_INVALID_ARG, "t=%d out of [0, %d)", t, cc->T);
    if (max_len < 0 || max_len > cc->Nmax)
        return fail(LOOPVQ_ERR_INVALID_ARG, "max_len=%d out of [0, Nmax=%d]", max_len, cc->Nmax);
    if (!std::isfinite(scale)) return fail(LOOPVQ_ERR_INVALID_ARG, "scale is not finite");
    if (scale <= 0.f) scale = 1.0f / std::sqrt((float)cc->D);
    const loopvq::DecodePlan plan = loopvq::plan_decode(*cc, max_len, true);
    if (plan.nsplit > 65535) return fail(LOOPVQ_ERR_UNSUPPORTED, "too many splits");
    if (!workspace || ws_bytes < plan.ws_bytes)
        return fail(LOOPVQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", plan.ws_bytes,
                    workspace ? ws_bytes : (size_t)0);
    if (!aligned16(workspace)) return fail(LOOPVQ_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    cudaError_t e = loopvq::launch_decode(*cc, plan, layer, t, q, nullptr, 0, lens, max_len, scale, out, lse,
                                          workspace, (cudaStream_t)stream, tq);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_tasq_decode_attn");
    return LOOPVQ_OK;
}

static loopvq_status check_window(const loopvq_window *w, const loopvq_cache *cc) {
    if (!w) return fail(LOOPVQ_ERR_INVALID_ARG, "window is NULL");
    LQ_TRY(check_shape(cc));
    if (loopvq::ncb_of(*cc) != 1)
        return fail(LOOPVQ_ERR_UNSUPPORTED, "the window's page encoder supports shared codebooks (ncb = 1) only");
    if (w->L != cc->L || w->T != cc->T || w->B != cc->B || w->Hkv != cc->Hkv || w->Hq != cc->Hq || w->D != cc->D)
        return fail(LOOPVQ_ERR_INVALID_ARG, "window shape (L, T, B, Hkv, Hq, D) differs from the cache's");
    if (w->n_sink <= 0 || w->n_recent <= 0 || w->n_sink % 8 != 0 || w->n_recent % 8 != 0)
        return fail(LOOPVQ_ERR_INVALID_ARG, "n_sink=%d, n_recent=%d must be positive multiples of 8", w->n_sink,
                    w->n_recent);
    // the page roll stages a (layer, loop step, sequence, head)'s n_recent recent slots in shared memory
    if ((size_t)w->n_recent * (size_t)w->D * 2 > kMaxOptinSmem)
        return fail(LOOPVQ_ERR_UNSUPPORTED, "n_recent=%d: %zu bytes of recent slots exceed the %zu bytes of shared "
                    "memory the page roll stages them in", w->n_recent, (size_t)w->n_recent * (size_t)w->D * 2,
                    kMaxOptinSmem);
    LQ_TRY(check_ptr(w->k_rot, "k_rot"));
    LQ_TRY(check_ptr(w->k_pre, "k_pre"));
    LQ_TRY(check_ptr(w->v, "v"));
    if (!w->fill || !w->coded_end) return fail(LOOPVQ_ERR_INVALID_ARG, "fill or coded_end is NULL");
    if ((reinterpret_cast<uintptr_t>(w->fill) & 3u) || (reinterpret_cast<uintptr_t>(w->coded_end) & 3u))
        return fail(LOOPVQ_ERR_INVALID_ARG, "fill or coded_end not 4-byte aligned");
    return LOOPVQ_OK;
}

int loopvq_window_slots(const loopvq_window *w) {
    if (!w || w->n_sink <= 0 || w->n_recent <= 0 || w->n_sink % 8 || w->n_recent % 8) return 0;
    return loopvq::window_slots(*w);
}

loopvq_status loopvq_window_advance(const loopvq_window *w, const loopvq_cache *cc, void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_window(w, cc));
    LQ_TRY(check_ptr(cc->idx, "idx"));
    LQ_TRY(check_ptr(cc->codebook, "codebook"));
    cudaError_t e = loopvq::launch_window_advance(*w, *cc, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_window_advance");
    return LOOPVQ_OK;
}

loopvq_status loopvq_window_append(const loopvq_window *w, int layer, int t, const uint16_t *k_rot,
                                   const uint16_t *k_pre, const uint16_t *v, void *stream) {
    g_err[0] = 0;
    if (!w) return fail(LOOPVQ_ERR_INVALID_ARG, "window is NULL");
    if (w->n_sink <= 0 || w->n_recent <= 0 || w->n_sink % 8 || w->n_recent % 8 || w->B <= 0 || w->Hkv <= 0 ||
        (w->D != 64 && w->D != 128))
        return fail(LOOPVQ_ERR_INVALID_ARG, "invalid window shape");
    if (layer < 0 || layer >= w->L) return fail(LOOPVQ_ERR_INVALID_ARG, "layer=%d out of [0, %d)", layer, w->L);
    if (t < 0 || t >= w->T) return fail(LOOPVQ_ERR_INVALID_ARG, "t=%d out of [0, %d)", t, w->T);
    LQ_TRY(check_ptr(w->k_rot, "window k_rot"));
    LQ_TRY(check_ptr(w->k_pre, "window k_pre"));
    LQ_TRY(check_ptr(w->v, "window v"));
    if (!w->fill) return fail(LOOPVQ_ERR_INVALID_ARG, "fill is NULL");
    LQ_TRY(check_ptr(k_rot, "k_rot"));
    LQ_TRY(check_ptr(k_pre, "k_pre"));
    LQ_TRY(check_ptr(v, "v"));
    cudaError_t e = loopvq::launch_window_append(*w, layer, t, k_rot, k_pre, v, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_window_append");
    return LOOPVQ_OK;
}

size_t loopvq_window_workspace_bytes(const loopvq_window *w, const loopvq_cache *cc, int max_coded) {
    if (check_window(w, cc) != LOOPVQ_OK || max_coded < 0 || max_coded > cc->Nmax) return 0;
    return loopvq::window_ws_bytes(*w, *cc, max_coded);
}

static loopvq_status window_decode(const char *name, const loopvq_window *w, const loopvq_cache *cc, int layer, int t,
                                   const uint16_t *k_rot, const uint16_t *k_pre, const uint16_t *v, const uint16_t *q,
                                   int max_coded, float scale, float *out, float *lse, void *workspace, size_t ws_bytes,
                                   void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_window(w, cc));
    LQ_TRY(check_ptr(cc->idx, "idx"));
    LQ_TRY(check_ptr(cc->slices, "slices"));
    LQ_TRY(check_ptr(cc->rope, "rope"));
    LQ_TRY(check_ptr(q, "q"));
    LQ_TRY(check_ptr(out, "out"));
    if (k_rot || k_pre || v) {
        LQ_TRY(check_ptr(k_rot, "k_rot"));
        LQ_TRY(check_ptr(k_pre, "k_pre"));
        LQ_TRY(check_ptr(v, "v"));
    }
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(LOOPVQ_ERR_INVALID_ARG, "lse not 4-byte aligned");
    if (layer < 0 || layer >= cc->L) return fail(LOOPVQ_ERR_INVALID_ARG, "layer=%d out of [0, %d)", layer, cc->L);
    if (t < 0 || t >= cc->T) return fail(LOOPVQ_ERR_INVALID_ARG, "t=%d out of [0, %d)", t, cc->T);
    if (max_coded < 0 || max_coded > cc->Nmax)
        return fail(LOOPVQ_ERR_INVALID_ARG, "max_coded=%d out of [0, Nmax=%d]", max_coded, cc->Nmax);
    if (!std::isfinite(scale)) return fail(LOOPVQ_ERR_INVALID_ARG, "scale is not finite");
    if (scale <= 0.f) scale = 1.0f / std::sqrt((float)cc->D);
    const size_t need = loopvq::window_ws_bytes(*w, *cc, max_coded);
    if (!workspace || ws_bytes < need)
        return fail(LOOPVQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? ws_bytes : (size_t)0);
    if (!aligned16(workspace)) return fail(LOOPVQ_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    cudaError_t e = loopvq::launch_window_decode(*w, *cc, layer, t, q, max_coded, scale, out, lse, workspace,
                                                 (cudaStream_t)stream, k_rot, k_pre, v);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return LOOPVQ_OK;
}

loopvq_status loopvq_window_decode_attn(const loopvq_window *w, const loopvq_cache *cc, int layer, int t,
                                        const uint16_t *q, int max_coded, float scale, float *out, float *lse,
                                        void *workspace, size_t ws_bytes, void *stream) {
    return window_decode("loopvq_window_decode_attn", w, cc, layer, t, nullptr, nullptr, nullptr, q, max_coded, scale,
                         out, lse, workspace, ws_bytes, stream);
}

loopvq_status loopvq_window_append_decode_attn(const loopvq_window *w, const loopvq_cache *cc, int layer, int t,
                                               const uint16_t *k_rot, const uint16_t *k_pre, const uint16_t *v,
                                               const uint16_t *q, int max_coded, float scale, float *out, float *lse,
                                               void *workspace, size_t ws_bytes, void *stream) {
    if (!k_rot || !k_pre || !v) {
        g_err[0] = 0;
        return fail(LOOPVQ_ERR_INVALID_ARG, "k_rot, k_pre and v are required");
    }
    return window_decode("loopvq_window_append_decode_attn", w, cc, layer, t, k_rot, k_pre, v, q, max_coded, scale,
                         out, lse, workspace, ws_bytes, stream);
}

loopvq_status loopvq_dequant_debug(const loopvq_cache *cc, int layer, int t, int kv, int b, int tok0, int ntok,
                                   int apply_rope, float *out, void *stream) {
    g_err[0] = 0;
    LQ_TRY(check_shape(cc));
    LQ_TRY(check_ptr(cc->idx, "idx"));
    LQ_TRY(check_ptr(cc->slices, "slices"));
    LQ_TRY(check_ptr(cc->rope, "rope"));
    if (layer < 0 || layer >= cc->L) return fail(LOOPVQ_ERR_INVALID_ARG, "layer=%d out of [0, %d)", layer, cc->L);
    if (t < 0 || t >= cc->T) return fail(LOOPVQ_ERR_INVALID_ARG, "t=%d out of [0, %d)", t, cc->T);
    if (kv != 0 && kv != 1) return fail(LOOPVQ_ERR_INVALID_ARG, "kv=%d (0 = keys, 1 = values)", kv);
    if (b < 0 || b >= cc->B) return fail(LOOPVQ_ERR_INVALID_ARG, "b=%d out of [0, %d)", b, cc->B);
    if (tok0 < 0 || ntok < 0 || tok0 + ntok > cc->Nmax)
        return fail(LOOPVQ_ERR_INVALID_ARG, "token range [%d, %d) outside [0, %d)", tok0, tok0 + ntok, cc->Nmax);
    if (ntok == 0) return LOOPVQ_OK;
    if (!out) return fail(LOOPVQ_ERR_INVALID_ARG, "out is NULL");
    cudaError_t e = loopvq::launch_dequant(*cc, layer, t, kv, b, tok0, ntok, apply_rope, out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "loopvq_dequant_debug");
    return LOOPVQ_OK;
}

const char *loopvq_last_error(void) { return g_err; }

int loopvq_abi_version(void) { return 3; }

}  // extern "C"
