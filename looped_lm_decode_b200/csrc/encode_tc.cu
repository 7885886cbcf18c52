// Encode on the 5th-generation tensor cores (tcgen05): nearest codebook entry as a distance contraction.
//
// LoopVQ paper, Sec. 4.3 "Encoding": a block is encoded by computing the distances to all
// codebook entries as a matrix product on tensor cores, then selecting the nearest entry;
// Sec. 4.1 eq. (4) for the coupled vectors, Sec. 2 eq. (2) for the nearest-entry rule.
//
// ||z - e_r||^2 = ||z||^2 - 2 (z.e_r - ||e_r||^2 / 2), so the nearest entry maximises
// s_r = z.e_r - h_r with h_r = ||e_r||^2 / 2.  The contraction computes s directly: every
// coupled vector is extended with three ones and every entry with -h_r split exactly into three
// bf16 parts, so one bf16 MMA (fp32 accumulate) per 16 coordinates yields s in tensor memory and the
// epilogue is a plain arg-max (first maximum, i.e. lowest index on ties) per TMEM lane.
//
// Tile: M = 128 coupled vectors (TOKS tokens x D/c channel groups of one sequence and KV head) by
// N = 256 entries; keys and values are two MMAs into the same 256 TMEM columns in turn.  With one
// codebook per channel group (PG) a tile is 128 tokens of one channel group, whose codebook is the B
// operand, and each tile writes its group's bytes of the index words.  Operands are
// staged in shared memory in the canonical K-major layout without swizzle: 8-row x 16-byte core
// matrices, the K-direction neighbour 128 bytes on (leading byte offset), the next 8 rows KB*128
// bytes on (stride byte offset).  One thread issues the MMAs and commits to an mbarrier; every wait
// on it is bounded in time (loopvq_set_wait_limit_ns); a CTA whose wait runs out sets the fault word
// that loopvq_fault_check reports, waits (bounded) for the work it already issued, writes 0xFF code bytes
// for its unfinished tokens and releases its tensor memory.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "loopvq_internal.cuh"

namespace loopvq {

namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// SWIZZLE_NONE K-major shared-memory matrix descriptor (tcgen05 format, version 1)
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;          // version
    return d;                         // base offset 0, lbo mode 0, layout type 0 (no swizzle)
}

// kind::f16 instruction descriptor: D fp32, A and B bf16, both K-major, M x N
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t mbar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(mbar), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Non-blocking test of the mbarrier phase (try_wait may suspend the thread for a while first).
__device__ __forceinline__ bool mbar_test(uint32_t mbar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(mbar), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for the mbarrier phase with the given parity; false once limit_ns have passed.  A limit of 0
// tests the phase once without blocking.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t mbar, uint32_t parity, uint64_t limit_ns) {
    if (limit_ns == 0) return mbar_test(mbar, parity);
    if (mbar_try(mbar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try(mbar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) return false;
    }
}

// Bound on the wait for work already issued, before a CTA that gave up releases its tensor memory.
constexpr uint64_t kDrainNs = 2000000000ull;

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
          "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
          "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}

// Wait for this thread's outstanding tcgen05.ld; the registers are named so that no read of them can be
// scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&v)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                   "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                   "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

// Exact arg-max of a TMEM lane's scores in two passes over the same columns.  Pass 1 takes the maximum
// M with three-input max.  Pass 2 finds the first column whose score is >= M (so == M): in each run of
// 32 columns, column j adds set(s_j >= M) * 2^-(j mod 32) to one of two accumulators of 16 columns, so
// each accumulator is an exact sum of distinct powers of two whose exponent names its lowest hit.
__device__ __forceinline__ float max3f(float x, float y, float z) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(x), "f"(y), "f"(z));
    return r;
}

__device__ __forceinline__ float ge_one(float x, float m) {      // 1.0f if x >= m, else 0.0f
    float r;
    asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(x), "f"(m));
    return r;
}

// maximum of NCOLS columns from column col0 (64 columns per wait)
template <int NCOLS>
__device__ __forceinline__ float cols_max(uint32_t taddr, int col0) {
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, m2 = -CUDART_INF_F, m3 = -CUDART_INF_F;
#pragma unroll 1
    for (int c = 0; c < NCOLS; c += 64) {
        uint32_t va[32], vb[32];
        tmem_ld32(taddr + col0 + c, va);
        tmem_ld32(taddr + col0 + c + 32, vb);
        tmem_wait_ld(va);
        tmem_wait_ld(vb);
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            m0 = max3f(m0, __uint_as_float(va[j]), __uint_as_float(va[j + 1]));
            m1 = max3f(m1, __uint_as_float(va[j + 2]), __uint_as_float(va[j + 3]));
            m2 = max3f(m2, __uint_as_float(vb[j]), __uint_as_float(vb[j + 1]));
            m3 = max3f(m3, __uint_as_float(vb[j + 2]), __uint_as_float(vb[j + 3]));
        }
    }
    return max3f(m0, m1, fmaxf(m2, m3));
}

// first of 32 columns (from c0) with score >= M, or -1
__device__ __forceinline__ int first_hit32(const uint32_t (&v)[32], float M, int c0) {
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        acc0 = fmaf(ge_one(__uint_as_float(v[j]), M), __int_as_float((127 - j) << 23), acc0);
        acc1 = fmaf(ge_one(__uint_as_float(v[16 + j]), M), __int_as_float((127 - 16 - j) << 23), acc1);
    }
    const float r = fmaxf(acc0, acc1);       // 0, or in [2^-31, 2): exponent 127 - (lowest hit)
    return r > 0.f ? c0 + 127 - (int)(__float_as_uint(r) >> 23) : -1;
}

// first of NCOLS columns from col0 with score >= M, or -1
template <int NCOLS>
__device__ __forceinline__ int cols_first(uint32_t taddr, int col0, float M) {
    int best = -1;
#pragma unroll 1
    for (int c = 0; c < NCOLS; c += 64) {
        uint32_t va[32], vb[32];
        tmem_ld32(taddr + col0 + c, va);
        tmem_ld32(taddr + col0 + c + 32, vb);
        tmem_wait_ld(va);
        tmem_wait_ld(vb);
        const int ia = first_hit32(va, M, col0 + c);
        const int ib = first_hit32(vb, M, col0 + c + 32);
        const int i = ia >= 0 ? ia : ib;
        if (best < 0) best = i;
    }
    return best;
}

}  // namespace tc

struct EncodeTcArgs {
    const uint16_t *xk, *xv;  // bf16, element (m, b - b0, n - tok0, h, d)
    int64_t s0, s1, s2, s3;
    uint32_t *idx;            // words of (layer, block, b = 0, h = 0)
    const uint16_t *cb;       // codebook of (layer, block, kv = 0, h = 0): [2][Hkv][K][G]
    int Hkv, K, Nmax, b0, nb, tok0, ntok;
    long long units_per_cta;  // flattened (head, [group,] sequence, tile) units, head-major, per CTA
    // TaSQ keys (TQ): weights of (layer, t = block Tc) [Tc][Hkv][D], order of (layer, block) [Hkv][D/2],
    // fp16 scales of (layer, t = block Tc) [Tc][B][Nmax]
    const float *tw;
    const int16_t *tperm;
    const uint16_t *tsig;
    int B;
    unsigned int *fault;      // per-GPU fault word: kFaultEncodeWait is set when a wait runs out
    unsigned long long wait_ns;
};

// Shared-memory plan (bytes): B operands for K and V (256 x KD bf16 each), A operands for K and V
// (128 x KD each), the code staging buffer, a per-row exchange area, the mbarrier and the TMEM address.
template <int KD>
struct TcSmem {
    static constexpr int kB = 256 * KD * 2;
    static constexpr int kA = 128 * KD * 2;
    static constexpr int offBK = 0;
    static constexpr int offBV = kB;
    static constexpr int offA = 2 * kB;                 // A operand of the keys
    static constexpr int offA2 = offA + kA;             // A operand of the values
    static constexpr int offCodes = offA2 + kA;         // 2 x 128 bytes
    static constexpr int offRed = offCodes + 256;       // per-row exchange: [2][128] float, [2][128] int
    static constexpr int offMbar = offRed + 2048;
    static constexpr int offTmem = offMbar + 8;
    static constexpr int kUsed = offTmem + 8;
    // at least 80 KiB keeps at most two CTAs per SM: 2 x 256 TMEM columns
    static constexpr int kAlloc = kUsed <= 80 * 1024 ? 80 * 1024 : ((kUsed + 1023) / 1024) * 1024;
};

// Threads: 256.  Thread (half, row) owns tile row `row` (= its TMEM lane, row = tid % 128): it stages
// the row's key (half 0) or value (half 1) coupled vector, and takes the arg-max over TMEM columns
// [128 * half, 128 * half + 128); the two halves combine through shared memory.
// TQ: keys coded after the TaSQ transform (LoopVQ paper, App. B): the key rows are the coupled vectors of
// TaSQ groups, u = fl(fl(w k) / sigma) in fp32 at the permuted channels, each split exactly into three
// bf16 parts (hi, mid, lo) along the contraction, against the entry repeated three times; values are
// coded plainly.  Key codes of TaSQ groups 2p and 2p + 1 go to bytes 0 and 1 of word p.
template <int D, int C, int TC, bool PG, bool TQ = false>
__global__ void __launch_bounds__(256, 2) encode_tc_kernel(const EncodeTcArgs a) {
    constexpr int G = C * TC;
    constexpr int KD = (((TQ ? 3 * G : G) + 3 + 15) / 16) * 16;   // contraction length: coordinates + 3, padded
    constexpr int KB = KD / 8;                          // 16-byte k-blocks per row
    constexpr int NG = D / C;                           // channel groups per token
    constexpr int NP = NG / 2;
    constexpr int TOKS = PG ? 128 : 128 / NG;           // tokens per 128-row tile
    constexpr int NGU = PG ? NG : 1;                    // channel groups in the unit space
    using S = TcSmem<KD>;
    static_assert(128 % NG == 0, "tile rows");
    static_assert(S::kUsed <= S::kAlloc, "shared memory plan");

    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, half = tid >> 7;
    const uint32_t mbar = tc::smem_u32(smem + S::offMbar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::offTmem);
    uint8_t *codes = smem + S::offCodes;
    float *red_m = reinterpret_cast<float *>(smem + S::offRed);
    int *red_i = reinterpret_cast<int *>(smem + S::offRed + 1024);

    // ---- TMEM (256 columns) and the mbarrier
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc::smem_u32(tmem_slot)),
                     "r"(256));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        tc::mbar_init(mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    // ---- B operands of head h (and group gq with PG): entry r -> [e_r (G coords), -h_hi, -h_mid, -h_lo,
    // 0 ...], h_r = ||e_r||^2 / 2
    auto build_b = [&](int h, int gq) {
        for (int it = tid; it < 2 * 256; it += 256) {
            const int kv = it >> 8, r = it & 255;
            uint16_t rw[KD];
#pragma unroll
            for (int k = 0; k < KD; ++k) rw[k] = 0;
            const int rep = (TQ && kv == 0) ? 3 : 1;       // TaSQ key rows: the entry against hi, mid, lo
            if (r < a.K) {
                const uint16_t *e = a.cb + (((size_t)kv * a.Hkv + h) * NGU + gq) * (size_t)a.K * G + (size_t)r * G;
                double hh = 0.0;
#pragma unroll
                for (int k = 0; k < G; ++k) {
                    rw[k] = e[k];
                    if constexpr (TQ) {
                        if (rep == 3) {
                            rw[G + k] = e[k];
                            rw[2 * G + k] = e[k];
                        }
                    }
                    const double v = (double)bf16_to_f32(e[k]);
                    hh += v * v;
                }
                hh *= 0.5;
                const float p1 = __bfloat162float(__float2bfloat16_rn((float)hh));
                const double r1 = hh - (double)p1;
                const float p2 = __bfloat162float(__float2bfloat16_rn((float)r1));
                const double r2 = r1 - (double)p2;
                rw[rep * G] = tc::bf16_bits_rn(-p1);
                rw[rep * G + 1] = tc::bf16_bits_rn(-p2);
                rw[rep * G + 2] = tc::bf16_bits_rn((float)-r2);
            } else {
                rw[rep * G] = tc::bf16_bits_rn(-1.0e30f);  // entries past K never win
            }
            unsigned char *base = smem + (kv ? S::offBV : S::offBK) + ((r >> 3) * KB) * 128 + (r & 7) * 16;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                uint4 v;
                v.x = rw[kb * 8 + 0] | ((uint32_t)rw[kb * 8 + 1] << 16);
                v.y = rw[kb * 8 + 2] | ((uint32_t)rw[kb * 8 + 3] << 16);
                v.z = rw[kb * 8 + 4] | ((uint32_t)rw[kb * 8 + 5] << 16);
                v.w = rw[kb * 8 + 6] | ((uint32_t)rw[kb * 8 + 7] << 16);
                *reinterpret_cast<uint4 *>(base + kb * 128) = v;
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
    };

    // ---- this CTA's run of units u = ((h * NGU + gq) * nb + brel) * ntiles + tile, walked without divisions
    const long long ntiles = (a.ntok + TOKS - 1) / TOKS;
    const long long total = ntiles * a.nb * a.Hkv * NGU;
    const long long u_begin = (long long)blockIdx.x * a.units_per_cta;
    const long long u_end = u_begin + a.units_per_cta < total ? u_begin + a.units_per_cta : total;
    struct Pos {
        int h, gq, brel, tile;
    };
    Pos cur;
    {
        const long long hb = u_begin / ntiles;
        cur.tile = (int)(u_begin - hb * ntiles);
        const long long hg = hb / a.nb;
        cur.brel = (int)(hb - hg * a.nb);
        cur.h = (int)(hg / NGU);
        cur.gq = (int)(hg - (long long)cur.h * NGU);
    }
    auto advance = [&](Pos &p) {
        if (++p.tile == (int)ntiles) {
            p.tile = 0;
            if (++p.brel == a.nb) {
                p.brel = 0;
                if (++p.gq == NGU) {
                    p.gq = 0;
                    ++p.h;
                }
            }
        }
    };

    int cur_h = cur.h, cur_g = cur.gq;
    build_b(cur_h, cur_g);                                 // also publishes the TMEM address
    const uint32_t tmem = *tmem_slot;

    const uint32_t idesc = tc::idesc_bf16(128, 256);
    const uint32_t bkaddr = tc::smem_u32(smem + S::offBK), bvaddr = tc::smem_u32(smem + S::offBV);
    uint32_t phase = 0;
    bool ok = true;
    const int rtok = PG ? row : row / NG, rg = PG ? 0 : row % NG;

    // this thread's coupled vector (key for half 0, value for half 1) of the next unit, one unit ahead:
    // bf16 bits, or with TaSQ keys the fp32 bits of u.  With TaSQ keys and G <= 16 (DEFER) the row holds
    // the raw key channels at the permuted positions and sgn the token's sigma of each loop step instead;
    // u is formed when the A operand is built, so the loads stay in flight across the current unit's
    // arg-max rather than stalling on the division here (at G = 32 the registers are not there).
    constexpr bool DEFER = TQ && G <= 16;
    uint32_t zn[G];
    float sgn[DEFER ? TC : 1];
    auto load_row = [&](bool valid, const Pos &p, uint32_t (&z)[G]) {
        const int nrel = p.tile * TOKS + rtok;
#pragma unroll
        for (int k = 0; k < G; ++k) z[k] = 0;
        if constexpr (DEFER) {
#pragma unroll
            for (int m = 0; m < TC; ++m) sgn[m] = 1.f;     // rows past the range: u = 0, no 0/0
        }
        if (valid && nrel < a.ntok) {
            if (TQ && half == 0) {
                // TaSQ group rg: channel i is the low (i even) or high (i odd) channel of pair perm[rg C/2 + i/2]
                const uint16_t *x = a.xk + (size_t)p.brel * a.s1 + (size_t)nrel * a.s2 + (size_t)p.h * a.s3;
                const int16_t *pm = a.tperm + (size_t)p.h * (D / 2) + rg * (C / 2);
#pragma unroll
                for (int i = 0; i < C; ++i) {
                    const int lowf = __ldg(pm + i / 2) & (D / 2 - 1);
                    const int f = (i & 1) ? lowf + D / 2 : lowf;
#pragma unroll
                    for (int m = 0; m < TC; ++m) {
                        if constexpr (DEFER) {
                            z[i * TC + m] = __ldg(x + (size_t)m * a.s0 + f);
                        } else {
                            const float wt = __ldg(a.tw + ((size_t)m * a.Hkv + p.h) * D + f);
                            const float sg = __half2float(__ushort_as_half(
                                __ldg(a.tsig + ((size_t)m * a.B + a.b0 + p.brel) * a.Nmax + a.tok0 + nrel)));
                            const float k = bf16_to_f32(__ldg(x + (size_t)m * a.s0 + f));
                            z[i * TC + m] = __float_as_uint(__fdiv_rn(__fmul_rn(wt, k), sg));
                        }
                    }
                }
                if constexpr (DEFER) {
#pragma unroll
                    for (int m = 0; m < TC; ++m)
                        sgn[m] = __half2float(__ushort_as_half(
                            __ldg(a.tsig + ((size_t)m * a.B + a.b0 + p.brel) * a.Nmax + a.tok0 + nrel)));
                }
            } else {
                const uint16_t *x = (half ? a.xv : a.xk) + (size_t)p.brel * a.s1 + (size_t)nrel * a.s2 +
                                    (size_t)p.h * a.s3 + (PG ? p.gq : rg) * C;
#pragma unroll
                for (int m = 0; m < TC; ++m)
#pragma unroll
                    for (int i = 0; i < C; ++i) z[i * TC + m] = __ldg(x + (size_t)m * a.s0 + i);
            }
        }
    };
    load_row(u_begin < u_end, cur, zn);

    for (long long u = u_begin; u < u_end; ++u) {
        const int tile = cur.tile, brel = cur.brel, h = cur.h, gq = cur.gq;
        advance(cur);
        if (h != cur_h || gq != cur_g) {                   // previous MMAs have completed: B may be rewritten
            build_b(h, gq);
            cur_h = h;
            cur_g = gq;
        }
        // ---- A operand of this thread's half: the coupled vector extended by three ones
        {
            uint16_t zr[KD];
            if (TQ && half == 0) {
                // u = fl(fl(w k) / sigma) at the permuted channels (DEFER: formed here), then
                // u = hi + mid + lo exactly (three round-to-nearest bf16 parts of an fp32 value)
                const int16_t *pm = a.tperm + (size_t)h * (D / 2) + rg * (C / 2);
#pragma unroll
                for (int k = 0; k < KD; ++k) zr[k] = 0;
#pragma unroll
                for (int i = 0; i < C; ++i) {
                    int f = 0;
                    if constexpr (DEFER) {
                        const int lowf = __ldg(pm + i / 2) & (D / 2 - 1);
                        f = (i & 1) ? lowf + D / 2 : lowf;
                    }
#pragma unroll
                    for (int m = 0; m < TC; ++m) {
                        const int k = i * TC + m;
                        float u;
                        if constexpr (DEFER) {
                            const float wt = __ldg(a.tw + ((size_t)m * a.Hkv + h) * D + f);
                            u = __fdiv_rn(__fmul_rn(wt, bf16_to_f32((uint16_t)zn[k])), sgn[m]);
                        } else {
                            u = __uint_as_float(zn[k]);
                        }
                        const uint16_t p1 = tc::bf16_bits_rn(u);
                        const float r1 = u - bf16_to_f32(p1);
                        const uint16_t p2 = tc::bf16_bits_rn(r1);
                        const float r2 = r1 - bf16_to_f32(p2);
                        zr[k] = p1;
                        zr[G + k] = p2;
                        zr[2 * G + k] = tc::bf16_bits_rn(r2);
                    }
                }
                zr[3 * G] = zr[3 * G + 1] = zr[3 * G + 2] = 0x3F80;   // bf16 1.0
            } else {
#pragma unroll
                for (int k = 0; k < KD; ++k) zr[k] = k < G ? (uint16_t)zn[k] : 0;
                zr[G] = zr[G + 1] = zr[G + 2] = 0x3F80;           // bf16 1.0
            }
            unsigned char *base = smem + (half ? S::offA2 : S::offA) + ((row >> 3) * KB) * 128 + (row & 7) * 16;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                uint4 v;
                v.x = zr[kb * 8 + 0] | ((uint32_t)zr[kb * 8 + 1] << 16);
                v.y = zr[kb * 8 + 2] | ((uint32_t)zr[kb * 8 + 3] << 16);
                v.z = zr[kb * 8 + 4] | ((uint32_t)zr[kb * 8 + 5] << 16);
                v.w = zr[kb * 8 + 6] | ((uint32_t)zr[kb * 8 + 7] << 16);
                *reinterpret_cast<uint4 *>(base + kb * 128) = v;
            }
        }
        load_row(u + 1 < u_end, cur, zn);
#pragma unroll 1
        for (int kv = 0; kv < 2; ++kv) {
            tc::fence_async_smem();
            tc::tc_fence_before();
            __syncthreads();
            // ---- s = [z, 1, 1, 1] . [e, -h] for all 256 entries, into TMEM columns [0, 256)
            if (tid == 0) {
                tc::tc_fence_after();
                const uint32_t aaddr = tc::smem_u32(smem + (kv ? S::offA2 : S::offA));
                const uint32_t baddr = kv ? bvaddr : bkaddr;
#pragma unroll
                for (int ks = 0; ks < KD / 16; ++ks) {
                    const uint64_t ad = tc::smem_desc(aaddr + ks * 256, 128, KB * 128);
                    const uint64_t bd = tc::smem_desc(baddr + ks * 256, 128, KB * 128);
                    tc::mma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(mbar);
            }
            // every thread waits (bounded); the CTA continues only if all of them saw the MMAs complete
            ok = __syncthreads_and(tc::mbar_wait_bounded(mbar, phase, a.wait_ns) ? 1 : 0) != 0;
            if (!ok) {
                // give up: record the fault, and let the contraction already issued finish (bounded) before
                // its shared-memory operands and tensor memory are released
                if (tid == 0) {
                    atomicOr(a.fault, kFaultEncodeWait);
                    tc::mbar_wait_bounded(mbar, phase, tc::kDrainNs);
                }
                __syncthreads();
                break;
            }
            phase ^= 1u;
            tc::tc_fence_after();
            // ---- exact arg-max of the row: maximum over both halves, then the first column equal to it
            const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
            red_m[half * 128 + row] = tc::cols_max<128>(taddr, half * 128);
            __syncthreads();
            const float M = fmaxf(red_m[row], red_m[128 + row]);
            red_i[half * 128 + row] = tc::cols_first<128>(taddr, half * 128, M);
            tc::tc_fence_before();
            __syncthreads();                               // TMEM is free again
            if (half == 0) {
                // a row without a hit has only NaN scores; it takes entry 0
                const int i0 = red_i[row], i1 = red_i[128 + row];
                codes[kv * 128 + row] = (uint8_t)(i0 >= 0 ? i0 : (i1 >= 0 ? i1 : 0));
            }
        }
        __syncthreads();
        if constexpr (PG) {
            // ---- group gq's bytes of the index words: K code at byte gq / NP, V code at byte 2 + gq / NP
            const int nr = tile * TOKS + row;
            if (nr < a.ntok) {
                uint32_t *idx_bh = a.idx + ((size_t)(a.b0 + brel) * a.Hkv + h) * idx_words_per_bh(a.Nmax, D, C);
                uint8_t *wb = reinterpret_cast<uint8_t *>(idx_bh + idx_word(a.tok0 + nr, gq % NP, NP));
                wb[2 * half + gq / NP] = ok ? codes[half * 128 + row] : (uint8_t)0xFF;
            }
        } else if (tid < TOKS * NP) {
            // ---- pack {K p, K p+NP, V p, V p+NP} words and store them (sentinel words after a timeout)
            const int t = tid / NP, p = tid % NP;
            const int nr = tile * TOKS + t;
            if (nr < a.ntok) {
                // key bytes: groups p and p + NP, or with TaSQ keys TaSQ groups 2p and 2p + 1
                const int k0 = TQ ? 2 * p : p, k1 = TQ ? 2 * p + 1 : p + NP;
                const uint32_t w = ok ? ((uint32_t)codes[t * NG + k0] | ((uint32_t)codes[t * NG + k1] << 8) |
                                         ((uint32_t)codes[128 + t * NG + p] << 16) |
                                         ((uint32_t)codes[128 + t * NG + p + NP] << 24))
                                      : 0xFFFFFFFFu;
                uint32_t *idx_bh = a.idx + ((size_t)(a.b0 + brel) * a.Hkv + h) * idx_words_per_bh(a.Nmax, D, C);
                idx_bh[idx_word(a.tok0 + nr, p, NP)] = w;
            }
        }
        if (!ok) break;
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
}

template <int D, int C, int TC, bool PG, bool TQ = false>
static cudaError_t launch_tc_ct(const EncodeTcArgs &a0, cudaStream_t s) {
    constexpr int NG = D / C;
    constexpr int TOKS = PG ? 128 : 128 / NG;
    constexpr int KD = (((TQ ? 3 : 1) * C * TC + 3 + 15) / 16) * 16;
    EncodeTcArgs a = a0;
    auto k = encode_tc_kernel<D, C, TC, PG, TQ>;
    cudaError_t e = ensure_dynamic_smem((const void *)k, TcSmem<KD>::kAlloc);
    if (e != cudaSuccess) return e;
    // CTAs resident per SM, from the limits that bind here: shared memory, registers and tensor memory
    // (each CTA allocates 256 of the SM's 512 TMEM columns)
    int dev = 0, sms = 0, smem_sm = 0, resv = 0;
    cudaFuncAttributes fa{};
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&resv, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncGetAttributes(&fa, k)) != cudaSuccess) return e;
    const int by_smem = smem_sm / (TcSmem<KD>::kAlloc + (int)fa.sharedSizeBytes + resv);
    const int by_regs = 65536 / (((fa.numRegs + 7) / 8) * 8 * 256);
    int per_sm = by_smem < by_regs ? by_smem : by_regs;
    if (per_sm > 2) per_sm = 2;
    if (per_sm < 1) return cudaErrorNotSupported;
    // persistent grid: one wave of CTAs, each taking an equal run of the head-major units
    const long long ntiles = (a.ntok + TOKS - 1) / TOKS;
    const long long total = ntiles * a.nb * a.Hkv * (PG ? NG : 1);
    long long ctas = (long long)sms * per_sm;
    if (ctas > total) ctas = total;
    a.units_per_cta = (total + ctas - 1) / ctas;
    ctas = (total + a.units_per_cta - 1) / a.units_per_cta;
    k<<<(unsigned)ctas, 256, TcSmem<KD>::kAlloc, s>>>(a);
    return cudaGetLastError();
}

// Returns cudaErrorNotSupported when the shape has no tensor-core instantiation.
cudaError_t launch_encode_tc(const loopvq_cache &cc, int layer, int block, const void *xk, const void *xv,
                             const int64_t *strides, int b0, int nb, int tok0, int ntok, cudaStream_t s) {
    EncodeTcArgs a{};
    a.xk = reinterpret_cast<const uint16_t *>(xk);
    a.xv = reinterpret_cast<const uint16_t *>(xv);
    a.s0 = strides[0];
    a.s1 = strides[1];
    a.s2 = strides[2];
    a.s3 = strides[3];
    a.idx = cc.idx + idx_base(cc, layer, block, 0, 0);
    a.cb = cc.codebook + codebook_base(cc, layer, block, 0, 0);
    a.Hkv = cc.Hkv;
    a.K = cc.K;
    a.Nmax = cc.Nmax;
    a.b0 = b0;
    a.nb = nb;
    a.tok0 = tok0;
    a.ntok = ntok;
    a.wait_ns = wait_limit_ns();
    if (cudaError_t ef = fault_word_for_current_device(&a.fault); ef != cudaSuccess) return ef;
    if (ncb_of(cc) == 1) {
        if (cc.D == 128 && cc.c == 4 && cc.Tc == 4) return launch_tc_ct<128, 4, 4, false>(a, s);
        if (cc.D == 128 && cc.c == 8 && cc.Tc == 4) return launch_tc_ct<128, 8, 4, false>(a, s);
        if (cc.D == 128 && cc.c == 16 && cc.Tc == 1) return launch_tc_ct<128, 16, 1, false>(a, s);
        if (cc.D == 128 && cc.c == 32 && cc.Tc == 1) return launch_tc_ct<128, 32, 1, false>(a, s);
        if (cc.D == 64 && cc.c == 4 && cc.Tc == 4) return launch_tc_ct<64, 4, 4, false>(a, s);
        if (cc.D == 64 && cc.c == 8 && cc.Tc == 4) return launch_tc_ct<64, 8, 4, false>(a, s);
        if (cc.D == 64 && cc.c == 16 && cc.Tc == 1) return launch_tc_ct<64, 16, 1, false>(a, s);
        if (cc.D == 64 && cc.c == 32 && cc.Tc == 1) return launch_tc_ct<64, 32, 1, false>(a, s);
    } else if (ncb_of(cc) == cc.D / cc.c) {
        if (cc.D == 128 && cc.c == 4 && cc.Tc == 4) return launch_tc_ct<128, 4, 4, true>(a, s);
        if (cc.D == 128 && cc.c == 8 && cc.Tc == 4) return launch_tc_ct<128, 8, 4, true>(a, s);
        if (cc.D == 128 && cc.c == 16 && cc.Tc == 1) return launch_tc_ct<128, 16, 1, true>(a, s);
        if (cc.D == 64 && cc.c == 4 && cc.Tc == 4) return launch_tc_ct<64, 4, 4, true>(a, s);
        if (cc.D == 64 && cc.c == 8 && cc.Tc == 4) return launch_tc_ct<64, 8, 4, true>(a, s);
    }
    return cudaErrorNotSupported;
}

// TaSQ keys (the scales must already be written): returns cudaErrorNotSupported when the shape has no
// tensor-core instantiation.
cudaError_t launch_tasq_encode_tc(const loopvq_cache &cc, const loopvq_tasq &tq, int layer, int block, const void *xk,
                                  const void *xv, const int64_t *strides, int b0, int nb, int tok0, int ntok,
                                  cudaStream_t s) {
    if (ncb_of(cc) != 1) return cudaErrorNotSupported;
    const int NB = cc.T / cc.Tc;
    const int t0 = block * cc.Tc;
    EncodeTcArgs a{};
    a.xk = reinterpret_cast<const uint16_t *>(xk);
    a.xv = reinterpret_cast<const uint16_t *>(xv);
    a.s0 = strides[0];
    a.s1 = strides[1];
    a.s2 = strides[2];
    a.s3 = strides[3];
    a.idx = cc.idx + idx_base(cc, layer, block, 0, 0);
    a.cb = cc.codebook + codebook_base(cc, layer, block, 0, 0);
    a.Hkv = cc.Hkv;
    a.K = cc.K;
    a.Nmax = cc.Nmax;
    a.b0 = b0;
    a.nb = nb;
    a.tok0 = tok0;
    a.ntok = ntok;
    a.wait_ns = wait_limit_ns();
    if (cudaError_t ef = fault_word_for_current_device(&a.fault); ef != cudaSuccess) return ef;
    a.tw = tq.w + ((size_t)layer * cc.T + t0) * cc.Hkv * cc.D;
    a.tperm = tq.perm + ((size_t)layer * NB + block) * cc.Hkv * (cc.D / 2);
    a.tsig = tq.sigma + ((size_t)layer * cc.T + t0) * cc.B * cc.Nmax;
    a.B = cc.B;
    if (cc.D == 128 && cc.c == 4 && cc.Tc == 4) return launch_tc_ct<128, 4, 4, false, true>(a, s);
    if (cc.D == 128 && cc.c == 4 && cc.Tc == 2) return launch_tc_ct<128, 4, 2, false, true>(a, s);
    if (cc.D == 128 && cc.c == 8 && cc.Tc == 4) return launch_tc_ct<128, 8, 4, false, true>(a, s);
    if (cc.D == 64 && cc.c == 8 && cc.Tc == 4) return launch_tc_ct<64, 8, 4, false, true>(a, s);
    return cudaErrorNotSupported;
}

}  // namespace loopvq
