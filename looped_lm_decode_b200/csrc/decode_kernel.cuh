// Shared pieces of the split-K decode kernels over the loop-axis coded cache (LoopVQ paper, Sec. 4.3
// "Attention"): the kernel arguments, the tile space that every split kernel shares out among its CTAs
// and the partial-record numbering the merge relies on, and small device helpers.  The kernels are in
// decode_split.cuh (every shape), decode_mha.cuh (one query head per KV head), decode_gqa.cuh (four
// query heads per KV head) and decode_merge.cuh (the log-sum-exp merge).
#pragma once

#include <cuda_fp16.h>
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
    const int32_t *starts;   // [B] first attended token, or null for start_all
    float *ws_o;             // [piece][QPK][D]  unnormalised partial outputs, piece = segment + CTA
    float2 *ws_ml;           // [piece][QPK]     (reference max, sum) in log2 units
    float *out;              // [B][Hq][D]
    float *lse;              // [B][Hq] or null
    int B, Hkv, Hq, K, Nmax, max_len;
    int ncta;                // CTAs of the split kernel (its grid); the tile space is shared out evenly
    int start_all;           // first attended token of every sequence when starts is null
    const float *tw;         // TaSQ: channel weights of (layer, t) [Hkv][D]
    const int16_t *tperm;    // TaSQ: low-channel order of (layer, block) [Hkv][D/2]
    const uint16_t *tsig;    // TaSQ: fp16 token scales of (layer, t) [B][Nmax]
    const uint16_t *wk;      // bf16 window of (layer, t), or null: rotated keys [B][Hkv][W][D]
    const uint16_t *wv;      //   values [B][Hkv][W][D]
    const int32_t *wfill;    //   [B] slots in use
    int W;                   //   slots per (sequence, KV head)
    const uint16_t *nk;      // the token being appended, or null: rotated key [B][Hkv][D] (slot fill - 1)
    const uint16_t *nkp;     //   key before RoPE [B][Hkv][D]
    const uint16_t *nv;      //   value [B][Hkv][D]
    uint16_t *wk_w;          //   window arrays of (layer, t) it is written to: rotated keys,
    uint16_t *wkp_w;         //   keys before RoPE,
    uint16_t *wv_w;          //   values
    float qscale;            // scale * log2(e)
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 unpack2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

__device__ __forceinline__ uint2 lds64(const unsigned char *smem, uint32_t off) {
    return *reinterpret_cast<const uint2 *>(smem + off);
}

__device__ __forceinline__ uint32_t word_k(const uint4 &w, int k) {
    return k == 0 ? w.x : (k == 1 ? w.y : (k == 2 ? w.z : w.w));
}

// Per-thread asynchronous prefetch queue: each thread copies, and later reads, only its own 16-byte
// entries, so completion is tracked with its own commit groups and no CTA barrier is involved.
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_smem), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// 16-byte copy that reads `full ? 16 : 0` bytes from src and zero-fills the rest of the destination
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst_smem, const void *src, bool full) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src), "r"(full ? 16 : 0)
                 : "memory");
}

// two fp32 values rounded to bf16 and packed: hi_elem in the upper half, lo_elem in the lower
__device__ __forceinline__ uint32_t cvt_bf16x2(float hi_elem, float lo_elem) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi_elem), "f"(lo_elem));
    return r;
}

// d += A B, m16n8k16, bf16 operands, fp32 accumulators (warp-level tensor-core product)
__device__ __forceinline__ void mma_bf16_16816(float4 &d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d.x), "+f"(d.y), "+f"(d.z), "+f"(d.w)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Sum of the T partial scores of a lane over the NL lanes of its slot, scattered so that each lane
// ends with the full score of one token: log2(T) halving exchanges, then butterflies over the
// remaining lane bits.  The token a lane finishes is given by tile_token().
template <int T, int NL>
__device__ __forceinline__ float reduce_scatter(const float (&v)[T], int ls, unsigned mask) {
    static_assert(T == 4 || T == 8, "tile");
    float a[T / 2];
    constexpr int o1 = NL / 2;
    const bool b1 = (ls & o1) != 0;
#pragma unroll
    for (int i = 0; i < T / 2; ++i) {
        const float keep = b1 ? v[T / 2 + i] : v[i];
        const float send = b1 ? v[i] : v[T / 2 + i];
        a[i] = keep + __shfl_xor_sync(mask, send, o1);
    }
    float c[T / 4];
    constexpr int o2 = NL / 4;
    const bool b2 = (ls & o2) != 0;
#pragma unroll
    for (int i = 0; i < T / 4; ++i) {
        const float keep = b2 ? a[T / 4 + i] : a[i];
        const float send = b2 ? a[i] : a[T / 4 + i];
        c[i] = keep + __shfl_xor_sync(mask, send, o2);
    }
    float r;
    int obut;
    if constexpr (T == 8) {
        constexpr int o3 = NL / 8;
        const bool b3 = (ls & o3) != 0;
        const float keep = b3 ? c[1] : c[0];
        const float send = b3 ? c[0] : c[1];
        r = keep + __shfl_xor_sync(mask, send, o3);
        obut = NL / 16;
    } else {
        r = c[0];
        obut = NL / 8;
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1)
        if (o <= obut) r += __shfl_xor_sync(mask, r, o);
    return r;
}

template <int T, int NL>
__device__ __forceinline__ int tile_token(int ls) {
    int t = ((ls & (NL / 2)) ? T / 2 : 0) + ((ls & (NL / 4)) ? T / 4 : 0);
    if constexpr (T == 8) t += (ls & (NL / 8)) ? 1 : 0;
    return t;
}

template <int T, int NL>
__device__ __forceinline__ int tile_owner(int t) {          // a lane of the slot that finishes token t
    int l = ((t & (T / 2)) ? NL / 2 : 0) + ((t & (T / 4)) ? NL / 4 : 0);
    if constexpr (T == 8) l += (t & 1) ? NL / 8 : 0;
    return l;
}

// ---- the tile space.  Sequence b attends tokens [st_b, len_b); they are covered by 4-token tiles
// from st_b rounded down to a tile (the tile's earlier tokens are masked), so index-word loads stay
// 16-byte aligned.  A segment is one (KV head h, sequence b), numbered s = h * B + b, and the tiles of
// all segments are laid end to end in that order: T = Hkv * Tb tiles, Tb = sum over b of the tiles of
// b.  CTA c of the G = ncta CTAs takes tiles [c T / G, (c + 1) T / G), so every CTA gets the same
// number of tiles whatever the lengths.  The part of segment s inside CTA c is a piece; pieces follow
// a staircase in which s and c never decrease, so s + c numbers them without collision, and the
// pieces of segment s are those of the CTAs that hold its first through its last tile.
__device__ __forceinline__ int seq_tiles(const DecodeArgs &a, int b, int &base, int &st, int &len) {
    len = min(max(__ldg(a.lens + b), 0), a.max_len);
    st = min(max(a.starts ? __ldg(a.starts + b) : a.start_all, 0), len);
    base = st & ~3;
    return len > st ? (len - base + 3) >> 2 : 0;
}

__device__ __forceinline__ long long warp_sum64(long long v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Tiles per KV head, Tb, and the tiles of the sequences before b, Pb(b) (one warp).
__device__ __forceinline__ void head_tiles(const DecodeArgs &a, int lane, int b, long long &Tb, long long &Pb) {
    Tb = 0;
    Pb = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
        const int bb = b0 + lane;
        int base, st, len;
        const long long t = bb < a.B ? seq_tiles(a, bb, base, st, len) : 0;
        Tb += warp_sum64(t);
        Pb += warp_sum64(bb < b ? t : 0);
    }
}

// First tile of CTA c among T tiles shared by G CTAs.
__device__ __forceinline__ long long cta_first_tile(long long c, long long T, long long G) { return c * T / G; }

// The CTA that holds tile x: the largest c with floor(c T / G) <= x.
__device__ __forceinline__ long long cta_of_tile(long long x, long long T, long long G) {
    return ((x + 1) * G + T - 1) / T - 1;
}

// This CTA's tile range and the segment holding its first tile (one warp; lane 0 writes info):
// info = {first tile, end tile, first tile of that segment, (h << 32) | b}.
__device__ __forceinline__ void cta_range(const DecodeArgs &a, int lane, long long *info) {
    long long Tb, unused;
    head_tiles(a, lane, 0, Tb, unused);
    const long long T = Tb * a.Hkv, G = a.ncta;
    const long long x0 = cta_first_tile(blockIdx.x, T, G), x1 = cta_first_tile(blockIdx.x + 1, T, G);
    long long seg0 = 0, hb = 0;
    if (x0 < x1) {
        const long long h0 = x0 / Tb, r = x0 - h0 * Tb;
        long long carry = 0;
        for (int b0 = 0; b0 < a.B; b0 += 32) {
            const int bb = b0 + lane;
            int base, st, len;
            const long long t = bb < a.B ? seq_tiles(a, bb, base, st, len) : 0;
            long long inc = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            inc += carry;
            const unsigned hit = __ballot_sync(0xffffffffu, bb < a.B && inc > r);
            if (hit) {
                const int l = __ffs(hit) - 1;
                const long long incl = __shfl_sync(0xffffffffu, inc, l), tl = __shfl_sync(0xffffffffu, t, l);
                seg0 = h0 * Tb + incl - tl;
                hb = (h0 << 32) | (long long)(b0 + l);
                break;
            }
            carry = __shfl_sync(0xffffffffu, inc, 31);
        }
    }
    if (lane == 0) {
        info[0] = x0;
        info[1] = x0 < x1 ? x1 : x0;
        info[2] = seg0;
        info[3] = hb;
    }
}

}  // namespace loopvq
