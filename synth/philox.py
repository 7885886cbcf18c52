"""Counter-based random numbers for the seeded synthetic workloads.

Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and Shaw,
"Parallel random numbers: as easy as 1, 2, 3" (SC'11).  A 128-bit counter and a
64-bit key are mixed by ten rounds; each round multiplies two of the four
32-bit words by fixed odd constants, swaps the high and low halves of the
products across lanes, and XORs in the key, which is bumped by two Weyl
constants between rounds.  Because every output depends only on
(counter, key), any element of a workload can be regenerated on its own, which
is what lets a CPU checker rebuild exactly the slice of a multi-GB cache that
it checks.

This module holds no arithmetic of the quantisation method; it only makes
numbers.  The CUDA twin in ``synth/csrc/synth_gen.cu`` implements the same
definition and is checked against this file bit for bit.
"""
from __future__ import annotations

import numpy as np

# Multipliers and Weyl key increments of Philox4x32 (Salmon et al. 2011, Table 2).
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
ROUNDS = 10

_MASK32 = np.uint64(0xFFFFFFFF)
_SH32 = np.uint64(32)


def philox4x32(c0, c1, c2, c3, k0: int, k1: int, rounds: int = ROUNDS):
    """Philox4x32-R on broadcastable uint32 counter words; returns four uint32 arrays."""
    c0, c1, c2, c3 = (np.asarray(v, dtype=np.uint64) & _MASK32 for v in (c0, c1, c2, c3))
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    k0 = int(k0) & 0xFFFFFFFF
    k1 = int(k1) & 0xFFFFFFFF
    m0 = np.uint64(PHILOX_M0)
    m1 = np.uint64(PHILOX_M1)
    for _ in range(rounds):
        p0 = m0 * c0          # exact: both factors < 2^32
        p1 = m1 * c2
        hi0, lo0 = p0 >> _SH32, p0 & _MASK32
        hi1, lo1 = p1 >> _SH32, p1 & _MASK32
        n0 = hi1 ^ c1 ^ np.uint64(k0)
        n2 = hi0 ^ c3 ^ np.uint64(k1)
        c0, c1, c2, c3 = n0, lo1, n2, lo0
        k0 = (k0 + PHILOX_W0) & 0xFFFFFFFF
        k1 = (k1 + PHILOX_W1) & 0xFFFFFFFF
    return tuple(v.astype(np.uint32) for v in (c0, c1, c2, c3))


# Irwin-Hall sum of the eight 16-bit halves of one Philox block: mean 8*65535/2,
# variance 8*(65536^2-1)/12.  The centred integer is exact in fp32 and is scaled
# by one fp32 constant, so CPU and GPU get identical bits.
IH_TERMS = 8
IH_CENTER = IH_TERMS * 65535 // 2               # 262140
IH_SCALE = np.float32(1.0 / np.sqrt(IH_TERMS * (65536.0 ** 2 - 1.0) / 12.0))


def approx_normal_from_words(w0, w1, w2, w3):
    """fp32 approx-N(0,1) sample from one Philox output block (Irwin-Hall of 8 uint16)."""
    s = np.zeros(np.shape(w0), dtype=np.int64)
    for w in (w0, w1, w2, w3):
        w = w.astype(np.int64)
        s += (w & 0xFFFF) + (w >> 16)
    centred = (s - IH_CENTER).astype(np.float32)   # |centred| <= 262140 < 2^24: exact
    return (centred * IH_SCALE).astype(np.float32)


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
