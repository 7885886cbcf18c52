/*
 * loopvq.h -- C ABI of the LoopVQ hot path on B200 (sm_100a).
 *
 * LoopVQ codes a looped transformer's KV cache along the loop axis: a coupled
 * sub-vector takes the same c channels from each of the Tc loop steps of a
 * block, G = c*Tc elements, and is stored as the index of its nearest entry in
 * a K-entry codebook, b/G bits per element, one index shared by the Tc loop
 * steps.  Decode attention at loop step t reads the shared indices through
 * that step's slice of the codebook, applies RoPE to the rebuilt keys and runs
 * split-K online-softmax attention merged by log-sum-exp.
 *   LoopVQ paper ("LoopVQ: Sub 1-bit KV Cache Quantization for Looped
 *   Transformers"), Sec. 2 eq. (2); Sec. 4.1 eq. (4)-(5); Sec. 4.3
 *   "Cache layout", "Encoding", "Attention"; App. C.
 *
 * Conventions for every call:
 *   - Pointers named in loopvq_cache and every array argument are DEVICE
 *     memory owned by the caller, unless the argument says otherwise.  The
 *     library allocates nothing on any call.
 *   - Calls are asynchronous on the caller's CUDA stream (cudaStream_t passed
 *     as void*; NULL is the legacy default stream).  No call synchronises.
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns a status and launches nothing.  loopvq_last_error() then gives a
 *     message (thread-local, valid until the next call on this thread).
 *   - A CUDA launch error returns LOOPVQ_ERR_CUDA with the CUDA error string.
 *
 * Supported shapes: D in {64, 128}; c in {4, 8, 16, 32}; Tc in {1, 2, 4}
 * with G = c*Tc <= 32; 1 <= K <= 256; Hq a multiple of Hkv with Hq/Hkv in
 * {1, 2, 4, 8}; T a multiple of Tc; Nmax a multiple of 4.  Tc = 1 is plain
 * per-loop-step coding (CQ, Sec. 2), which runs on the same kernels.
 */
#ifndef LOOPVQ_H
#define LOOPVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LOOPVQ_OK = 0,
    LOOPVQ_ERR_INVALID_ARG = 1,   /* null pointer, out-of-range index or size */
    LOOPVQ_ERR_UNSUPPORTED = 2,   /* valid but not built: D, c, Tc, Hq/Hkv outside the supported set */
    LOOPVQ_ERR_WORKSPACE = 3,     /* workspace missing or smaller than loopvq_decode_workspace_bytes */
    LOOPVQ_ERR_CUDA = 4,          /* a launch failed; loopvq_last_error() holds the CUDA message */
    LOOPVQ_ERR_TIMEOUT = 5,       /* reported by loopvq_fault_check: an encode's bounded wait ran out */
    LOOPVQ_ERR_OVERFLOW = 6       /* reported by loopvq_fault_check: a window roll found the coded cache full */
} loopvq_status;

enum { LOOPVQ_BF16 = 0, LOOPVQ_FP32 = 1 };

/*
 * The coded cache of one model (all layers), described by shape and by four
 * caller-owned device buffers.  NB = T / Tc blocks, NP = D / (2c) pair-groups.
 *
 * idx       uint32 words, [L][NB][B][Hkv][Nmax/4][NP][4].  Word (token n,
 *           pair-group p) sits at tile n/4, slot n%4 and packs four 8-bit
 *           codes: byte0 = K code of channel group p, byte1 = K code of group
 *           p + NP (the group holding the RoPE partners of group p), byte2 =
 *           V code of group p, byte3 = V code of group p + NP.  Channel group
 *           g covers channels g*c .. g*c+c-1.  One word serves all Tc loop
 *           steps of its block (Sec. 4.3 "Cache layout": one index row per
 *           block).  2*D/c bytes per token, head and block.
 * codebook  bf16 [L][NB][2][Hkv][NCB][K][G], 2 = {K, V}; coordinate i*Tc + m
 *           of an entry belongs to channel i at loop step m of the block
 *           (eq. 4).  NCB = 1: one codebook per (layer, block, KV head, K|V),
 *           shared by all channel groups; NCB = D/c: one per channel group g
 *           (the paper's notation, eq. 5), set by the field ncb.
 * slices    bf16 [L][T][2][Hkv][K][NCB*c]: loop step t = beta*Tc + m keeps
 *           coordinates i*Tc + m, i < c, of every entry, code-major (row r
 *           holds entry r of every group's codebook) (Sec. 4.3 "Attention":
 *           the slice B_t, cut once when the model is loaded).  Written by
 *           loopvq_prepare.
 * rope      fp32 [Nmax][D]: row p holds cos(p*w_f) in [0, D/2) and sin(p*w_f)
 *           in [D/2, D), w_f = theta^(-2f/D), angles in fp64 (App. C: one row
 *           of D values per position).  Written by loopvq_prepare.
 */
typedef struct loopvq_cache {
    int32_t L, T, Tc, Hkv, Hq, D, c, K;
    int32_t B, Nmax;
    float theta;                 /* RoPE base, e.g. 1e4 */
    uint32_t *idx;
    const uint16_t *codebook;
    uint16_t *slices;
    float *rope;
    int32_t ncb;                 /* codebooks per (layer, block, KV head, K|V): 0 or 1 = shared, D/c = per group */
} loopvq_cache;

/* Element counts of the four buffers (0 if the shape is invalid). */
size_t loopvq_idx_words(const loopvq_cache *cache);
size_t loopvq_codebook_elems(const loopvq_cache *cache);
size_t loopvq_slice_elems(const loopvq_cache *cache);
size_t loopvq_rope_elems(const loopvq_cache *cache);

/*
 * Load-time preparation (Sec. 4.3 "Attention"; App. C): cut every loop
 * step's codebook slice from the codebooks, and fill the RoPE table.
 * Reads cache->codebook, writes cache->slices and cache->rope.
 */
loopvq_status loopvq_prepare(const loopvq_cache *cache, void *stream);

/*
 * Encode (Sec. 4.3 "Encoding"; eq. 2 and 4): for the sequences
 * b0 .. b0+nb-1 and tokens tok0 .. tok0+ntok-1, build every coupled vector of
 * block `block` of layer `layer` for keys and values and store the index of
 * its nearest codebook entry (squared Euclidean distance, lowest index on
 * ties) into cache->idx.
 *
 * xk, xv    pre-RoPE keys / values of the Tc loop steps of the block, dtype
 *           LOOPVQ_BF16 or LOOPVQ_FP32.  Element (m, b, n, h, d) is at
 *           x[m*s[0] + (b-b0)*s[1] + (n-tok0)*s[2] + h*s[3] + d]; strides s are
 *           in elements, d is contiguous.  Both use the same strides.
 * Only the words of the named sequences and tokens are written; every word
 * is rewritten whole (K and V codes of both groups of a pair).
 */
loopvq_status loopvq_encode(const loopvq_cache *cache, int layer, int block,
                            const void *xk, const void *xv, int x_dtype,
                            const int64_t x_strides[4],
                            int b0, int nb, int tok0, int ntok, void *stream);

/* Workspace bytes loopvq_decode_attn needs for caches of up to max_len tokens. */
size_t loopvq_decode_workspace_bytes(const loopvq_cache *cache, int max_len);

/*
 * Decode attention at loop step t (0-based) of layer `layer`
 * (Sec. 4.3 "Attention"; App. C):
 *   for every sequence b and query head hq (KV head hq / (Hq/Hkv)):
 *     k_n = RoPE(rebuilt key of token n, position n), v_n = rebuilt value,
 *     s_n = scale * <q, k_n>,  out = sum_n softmax(s)_n v_n,
 *     lse = ln sum_n exp(s_n),  over tokens n < len_b.
 * Tokens are cut into splits, each attended by its own thread blocks; the
 * splits are combined through their log-sum-exp, which is exact.
 *
 * q         bf16 [B][Hq][D], already rotated at the query position.
 * lens      int32 [B] device; each length is clamped to [0, max_len].
 * max_len   host-side upper bound of the lengths, 0 <= max_len <= Nmax.
 * scale     score scale; <= 0 selects 1/sqrt(D).
 * out       fp32 [B][Hq][D]; len_b == 0 gives zeros.
 * lse       fp32 [B][Hq] natural-log log-sum-exp, -inf for len_b == 0; may be NULL.
 * workspace device scratch of at least loopvq_decode_workspace_bytes(cache, max_len)
 *           bytes, 16-byte aligned; its contents on entry do not matter.  Calls
 *           that share a workspace must be ordered on the GPU (one stream, or
 *           events).
 */
loopvq_status loopvq_decode_attn(const loopvq_cache *cache, int layer, int t,
                                 const uint16_t *q, const int32_t *lens, int max_len,
                                 float scale, float *out, float *lse,
                                 void *workspace, size_t ws_bytes, void *stream);

/*
 * Decode attention over a token range of the coded cache (Sec. 4.3 "Cache
 * layout" and "Attention"): the same as loopvq_decode_attn, over tokens
 * start_b <= n < len_b.  This is the coded part of a cache whose first n_s
 * (sink) and last n_r (recent) tokens are kept in bf16.  Combine it with
 * loopvq_bf16_decode_attn over the bf16 tokens through loopvq_merge2.
 *
 * starts    int32 [B] device, or NULL for all 0; each start is clamped to
 *           [0, len_b].  Any start works: index words are read in 4-token tiles
 *           and the tile tokens before the start are masked.
 * Positions for RoPE stay absolute (token index n).  Workspace as for
 * loopvq_decode_attn.  len_b <= start_b gives zeros and lse = -inf.
 */
loopvq_status loopvq_decode_attn_range(const loopvq_cache *cache, int layer, int t,
                                       const uint16_t *q, const int32_t *starts, const int32_t *lens,
                                       int max_len, float scale, float *out, float *lse,
                                       void *workspace, size_t ws_bytes, void *stream);

/*
 * A bf16 KV cache: the unquantized layout that LoopVQ is compared against
 * (Sec. 5.3), and the store of the sink and recent tokens (Sec. 4.3 "Cache
 * layout").  Keys are stored as the model attends to them, already rotated
 * by RoPE at their positions.  Caller-owned device buffers:
 *   k, v      bf16 [B][Hkv][Nmax][D], 16-byte aligned.
 * D in {64, 128}; Hq a multiple of Hkv with Hq / Hkv in {1, 2, 4, 8}.
 */
typedef struct loopvq_bf16_cache {
    int32_t B, Hkv, Hq, D, Nmax;
    const uint16_t *k;
    const uint16_t *v;
} loopvq_bf16_cache;

/* Workspace bytes loopvq_bf16_decode_attn needs for up to max_len tokens per sequence. */
size_t loopvq_bf16_decode_workspace_bytes(const loopvq_bf16_cache *cache, int max_len);

/*
 * Decode attention over a bf16 cache (the bf16 kernel of Sec. 4.3
 * "Attention"): for every sequence b and query head hq (KV head
 * hq / (Hq/Hkv)), s_n = scale * <q, k_n>, out = sum_n softmax(s)_n v_n,
 * lse = ln sum_n exp(s_n), over tokens start_b <= n < len_b.  Split over
 * tokens and merged by log-sum-exp like loopvq_decode_attn.
 *
 * q         bf16 [B][Hq][D], rotated at the query position.
 * starts    int32 [B] device or NULL (all 0); lens int32 [B] device; both
 *           clamped as in loopvq_decode_attn_range.  max_len <= Nmax is a host
 *           upper bound of the lengths.
 * scale     <= 0 selects 1/sqrt(D).
 * out, lse, workspace as for loopvq_decode_attn.
 */
loopvq_status loopvq_bf16_decode_attn(const loopvq_bf16_cache *cache, const uint16_t *q,
                                      const int32_t *starts, const int32_t *lens, int max_len,
                                      float scale, float *out, float *lse,
                                      void *workspace, size_t ws_bytes, void *stream);

/*
 * Log-sum-exp merge of two attentions of the same queries over disjoint
 * token sets (Sec. 4.3 "Attention": the bf16 and the quantized kernels'
 * results are combined exactly):
 *   m = max(lse_a, lse_b), w_x = exp(lse_x - m),
 *   out = (w_a out_a + w_b out_b) / (w_a + w_b),  lse = m + ln(w_a + w_b).
 * A part with lse = -inf (no tokens) contributes nothing; both empty gives
 * zeros and -inf.
 *
 * out_a, out_b, out   fp32 [rows][D]; lse_a, lse_b, lse fp32 [rows] (lse may be
 * NULL).  out may alias out_a or out_b and lse may alias lse_a or lse_b.
 * D in {64, 128}.
 */
loopvq_status loopvq_merge2(const float *out_a, const float *lse_a, const float *out_b,
                            const float *lse_b, int rows, int D, float *out, float *lse,
                            void *stream);

/*
 * TaSQ applied before loop-axis coupling (App. B): keys are mapped to
 *   u = P(w (.) k / sigma)
 * before their coupled vectors are built, and rebuilt keys are mapped back
 * (k_hat = sigma * P^-1(u_hat) / w) before RoPE.  Values are not transformed.
 *   w      fp32 [L][T][Hkv][D]: channel weights of loop step t, layer and
 *          head; the two channels of a RoPE pair {f, f + D/2} must have the
 *          same weight (the post-RoPE query moment is pair-symmetric).
 *   perm   int16 [L][NB][Hkv][D/2]: the permutation P of (layer, block, KV
 *          head), as an order of the low channels 0 .. D/2-1.  Key code g
 *          (g < D/c) holds the c/2 RoPE pairs with low channels
 *          perm[g*c/2 + j], j < c/2, each as (f, f + D/2), at every loop step
 *          of the block: coordinate i*Tc + m is channel f of pair i/2 (even i)
 *          or its partner f + D/2 (odd i) at loop step m.
 *   sigma  fp16 [L][T][B][Nmax]: per-token scale of loop step t and layer,
 *          the root mean square of w (.) k over all KV heads and channels of
 *          the token, rounded to fp16; written by loopvq_tasq_encode.
 * With TaSQ the index word (token n, pair-group p) holds: byte0 = K code of
 * TaSQ group 2p, byte1 = K code of group 2p+1, byte2/3 = V codes of channel
 * groups p and p + NP as without TaSQ.  Caches used with TaSQ share one
 * codebook per (layer, block, KV head, K|V) (ncb = 1) and have c in {4, 8}.
 */
typedef struct loopvq_tasq {
    const float *w;
    const int16_t *perm;
    uint16_t *sigma;
} loopvq_tasq;

/* Elements of the three TaSQ buffers for a cache (0 if the cache cannot be used with TaSQ). */
size_t loopvq_tasq_w_elems(const loopvq_cache *cache);
size_t loopvq_tasq_perm_elems(const loopvq_cache *cache);
size_t loopvq_tasq_sigma_elems(const loopvq_cache *cache);

/*
 * loopvq_encode with TaSQ (App. B, eq. 10-11): for sequences b0 .. b0+nb-1
 * and tokens tok0 .. tok0+ntok-1 of every loop step of the block, compute
 * sigma (fp64 root mean square, rounded to fp16) into tasq->sigma, then code
 * the keys' coupled vectors of u and the values' coupled vectors (nearest
 * entries as in loopvq_encode, lowest index on ties; for bf16 input the fp32
 * u is split exactly into three bf16 parts, so the tensor-core products stay
 * exact).  Arguments as for loopvq_encode; the call must cover all KV heads
 * of the tokens (sigma spans them).
 */
loopvq_status loopvq_tasq_encode(const loopvq_cache *cache, const loopvq_tasq *tasq, int layer, int block,
                                 const void *xk, const void *xv, int x_dtype, const int64_t x_strides[4],
                                 int b0, int nb, int tok0, int ntok, void *stream);

/*
 * loopvq_decode_attn over a TaSQ-coded cache: k_n = RoPE(sigma_n *
 * P^-1(rebuilt u) / w, position n).  Arguments and workspace as for
 * loopvq_decode_attn.
 */
loopvq_status loopvq_tasq_decode_attn(const loopvq_cache *cache, const loopvq_tasq *tasq, int layer, int t,
                                      const uint16_t *q, const int32_t *lens, int max_len, float scale,
                                      float *out, float *lse, void *workspace, size_t ws_bytes, void *stream);

/*
 * The bf16 window of a coded cache and its decode-time life cycle (Sec. 4.3
 * "Cache layout": the first n_s (sink) and the most recent n_r tokens of a
 * request stay in bf16, pages of 8 tokens; "Encoding": during decode the
 * oldest recent page is encoded once the window holds 8 tokens more than n_r).
 *
 * Every sequence b has W = n_sink + n_recent + 8 slots per (layer, loop step):
 *   slots 0 .. n_sink-1        tokens 0 .. n_sink-1 (the sink, once filled);
 *   slots n_sink .. fill_b-1   tokens coded_end_b .. coded_end_b + fill_b - n_sink - 1
 *                              (the recent tokens, oldest first);
 * and the tokens n_sink <= n < coded_end_b are in the coded cache.  A token is
 * held twice as a key: rotated at its position (what attention reads) and
 * before RoPE (what the encoder reads when its page leaves the window, since
 * keys are coded before RoPE).  Caller-owned device buffers:
 *   k_rot, k_pre, v   bf16 [L][T][B][Hkv][W][D], 16-byte aligned;
 *   fill              int32 [B], slots in use (0 .. W);
 *   coded_end         int32 [B], >= n_sink; starts at n_sink for an empty
 *                     coded part.
 * Shapes L, T, B, Hkv, Hq, D must equal those of the coded cache used with it;
 * n_sink and n_recent are positive multiples of 8.  The caller fills the
 * window and the counters after prefill (loopvq_encode for the coded part).
 */
typedef struct loopvq_window {
    int32_t L, T, B, Hkv, Hq, D;
    int32_t n_sink, n_recent;
    uint16_t *k_rot;
    uint16_t *k_pre;
    uint16_t *v;
    int32_t *fill;
    int32_t *coded_end;
} loopvq_window;

/* Slots per (layer, loop step, sequence, KV head): n_sink + n_recent + 8 (0 if invalid). */
int loopvq_window_slots(const loopvq_window *w);

/*
 * Start a decode step: for every sequence whose window is full (fill_b == W)
 * encode its oldest recent page (slots n_sink .. n_sink+7, tokens coded_end_b
 * .. coded_end_b+7) for every layer and block from k_pre and v into the coded
 * cache (exact fp32 nearest entries, as loopvq_encode), move the remaining
 * recent slots down by 8 and set coded_end_b += 8, fill_b -= 8; then reserve
 * the new token's slot (fill_b += 1) for every sequence.  All decisions are
 * taken on the device from fill and coded_end; nothing synchronises.  A page
 * whose tokens would reach past the coded cache's Nmax is not written.
 */
loopvq_status loopvq_window_advance(const loopvq_window *w, const loopvq_cache *cache, void *stream);

/*
 * Write the current token of (layer, t) into slot fill_b - 1 of every
 * sequence: k_rot (rotated at its position), k_pre (before RoPE) and v are
 * bf16 [B][Hkv][D], 16-byte aligned.  Call after loopvq_window_advance.
 */
loopvq_status loopvq_window_append(const loopvq_window *w, int layer, int t, const uint16_t *k_rot,
                                   const uint16_t *k_pre, const uint16_t *v, void *stream);

/* Workspace bytes loopvq_window_decode_attn needs with coded parts of up to max_coded tokens. */
size_t loopvq_window_workspace_bytes(const loopvq_window *w, const loopvq_cache *cache, int max_coded);

/*
 * Decode attention of (layer, t) over the window and the coded cache: window
 * slots 0 .. fill_b-1 (keys stored rotated) and the coded tokens
 * n_sink <= n < coded_end_b, combined through their log-sum-exps (Sec. 4.3
 * "Attention").  Two launches: the coded split kernel, and its merge kernel,
 * which attends to the window slots while the split kernel finishes.
 * max_coded is a host upper bound of coded_end (<= Nmax).
 * q, scale, out, lse as for loopvq_decode_attn; workspace of at least
 * loopvq_window_workspace_bytes(w, cache, max_coded) bytes.
 */
loopvq_status loopvq_window_decode_attn(const loopvq_window *w, const loopvq_cache *cache, int layer, int t,
                                        const uint16_t *q, int max_coded, float scale, float *out,
                                        float *lse, void *workspace, size_t ws_bytes, void *stream);

/*
 * loopvq_window_append followed by loopvq_window_decode_attn, in the decode
 * call's two launches: the merge kernel writes the new token into slot
 * fill_b - 1 of (layer, t) (rotated key, key before RoPE, value, as
 * loopvq_window_append does) and attends to it together with the other
 * window slots.  Results and window contents equal those of the two calls.
 * k_rot, k_pre, v: bf16 [B][Hkv][D], 16-byte aligned, as for
 * loopvq_window_append; the other arguments as for loopvq_window_decode_attn.
 * Call after loopvq_window_advance; concurrent calls for the same (layer, t)
 * race on the window slot.
 */
loopvq_status loopvq_window_append_decode_attn(const loopvq_window *w, const loopvq_cache *cache, int layer, int t,
                                               const uint16_t *k_rot, const uint16_t *k_pre, const uint16_t *v,
                                               const uint16_t *q, int max_coded, float scale, float *out,
                                               float *lse, void *workspace, size_t ws_bytes, void *stream);

/*
 * Explicit reconstruction for checking (eq. 5): for sequence b, tokens
 * tok0 .. tok0+ntok-1 and every KV head, the loop-step-t reconstruction of
 * keys (kv = 0) or values (kv = 1); keys are rotated by RoPE at their
 * positions when apply_rope != 0.
 * out       fp32 [Hkv][ntok][D].
 */
loopvq_status loopvq_dequant_debug(const loopvq_cache *cache, int layer, int t, int kv,
                                   int b, int tok0, int ntok, int apply_rope,
                                   float *out, void *stream);

/*
 * Size in bytes of the built-in split scratch used by loopvq_decode_attn_noalloc.
 */
#define LOOPVQ_NOALLOC_SCRATCH_BYTES (8u << 20)
size_t loopvq_noalloc_scratch_bytes(void);

/*
 * Decode attention without any caller workspace.  (The LoopVQ paper has no
 * counterpart: this is a deployment convenience of this library.)
 *
 * Some callers cannot allocate device memory at all: plain C hosts with no
 * device allocator of their own, plug-ins whose host application owns every
 * byte of the device through its own allocator, and serving loops that must
 * not call cudaMalloc because it can synchronise the device.  This entry
 * point computes exactly what loopvq_decode_attn computes (same kernels, same
 * arguments minus the workspace) but keeps the split partials in a fixed
 * 8 MiB array compiled into the library (LOOPVQ_NOALLOC_SCRATCH_BYTES).
 *
 *  - Every GPU that loads the library holds that array until the process
 *    exits.  Nothing is allocated or freed by this call (no cudaMalloc, no
 *    cudaFree, no allocating library routine).
 *  - The first call on a device looks up the array's device address on the
 *    current device (cudaGetSymbolAddress) and caches it; make that first call
 *    before any stream capture.
 *  - A call whose split scratch, loopvq_decode_workspace_bytes(cache, max_len),
 *    exceeds the array is rejected with LOOPVQ_ERR_WORKSPACE and a message
 *    naming both sizes; nothing is launched.
 *  - All calls in the process share the one array per device and it keeps the
 *    last call's contents (no call needs it cleared: every partial that is read
 *    is written by the same call first).  Calls that overlap on the GPU, for
 *    example on two streams, race on it: issue them in order on one stream.
 */
loopvq_status loopvq_decode_attn_noalloc(const loopvq_cache *cache, int layer, int t,
                                         const uint16_t *q, const int32_t *lens, int max_len,
                                         float scale, float *out, float *lse, void *stream);

/* Message of the last failed call on this thread ("" if none). */
const char *loopvq_last_error(void);

/*
 * Faults found on the device.  Calls are asynchronous, so a kernel that cannot
 * finish its job cannot return an error from the call that launched it;
 * instead it sets a bit in a fault word that the library keeps on each GPU:
 *   - the tensor-core encoder (loopvq_encode and loopvq_tasq_encode with bf16
 *     input) bounds each wait for its own contraction; when the bound runs
 *     out it stops, waits (bounded by 2 s) for the work it already issued,
 *     releases its tensor memory, writes 0xFF code bytes for the tokens it
 *     had not finished and sets the fault;
 *   - loopvq_window_advance does not roll a sequence whose coded cache has no
 *     room for the page (coded_end + 8 > Nmax) and sets the fault; that
 *     sequence's window stays full, so its next append overwrites the newest
 *     slot.
 * loopvq_fault_check synchronises `stream` (the one call that does), reads
 * and clears the current GPU's fault word and returns LOOPVQ_ERR_TIMEOUT or
 * LOOPVQ_ERR_OVERFLOW (message in loopvq_last_error) or LOOPVQ_OK.  The word
 * is shared by every stream and thread of the process on that GPU; its first
 * use on a device looks up the word's address (make that first call before
 * any stream capture).
 *
 * loopvq_set_wait_limit_ns sets, for the whole process, the bound in
 * nanoseconds on each such wait of the encoder (default 2e9); 0 tests the
 * wait once without blocking and gives up if the work is not finished,
 * which tests use to exercise this path.
 * No page of the paper corresponds; it is the library's error channel.
 */
loopvq_status loopvq_fault_check(void *stream);
void loopvq_set_wait_limit_ns(uint64_t ns);
uint64_t loopvq_wait_limit_ns(void);

/* ABI version, bumped on any incompatible change. */
int loopvq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOOPVQ_H */
