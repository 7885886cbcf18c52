"""Seeded synthetic workloads shaped like the looped models the LoopVQ pages measure.

Five workload shapes (all K = 256 codes, b = 8 bits):

  tiny       1 layer, 1 KV head, T = 4, D = 64, c = 4 (G = 16), 256 tokens
  ctx4k      24 layers, 16 KV/16 q heads, T = 4, D = 128, c = 4, batch 32, 4096 tokens
  ctx32k     same model, batch 8, 32768-token cache, lengths uniform in [16384, 32768]
  gqa16k     24 layers, 4 KV/16 q heads, D = 128, c = 8 (G = 32, 0.25 bit), batch 64, 16384 tokens
  deep32     4 layers, 40 KV heads, T = 32 coded as 8 blocks of 4, D = 128, c = 4,
             batch 2, 8192 tokens
  ctx32k_cq  ctx32k coded per loop step (CQ: Tc = 1, c = G = 16, 0.5 bit), the
             baseline the pages compare LoopVQ against at the same bitwidth; same
             seed as ctx32k, so keys, values, queries and lengths are identical
  ctx32k_pg  ctx32k with one codebook per channel group (32 per head and K|V),
             the paper's notation; same seed as ctx32k
  ctx32k_tasq  ctx32k with keys coded after the TaSQ transform (seeded weights
             and pair permutations); same seed as ctx32k

The model shapes follow the pages' Ouro-1.4B description (24 layers, 16 heads of
dimension 128, 4 loop steps) and the deep-recurrence variant follows the
32-iteration Huginn setting coded in blocks of four (LoopVQ paper, Sec. 5.1
"Models" and "Methods").

Pre-RoPE keys and values follow a loop-axis AR(1) process, which mimics the
strong adjacent-loop correlation the pages report (LoopVQ paper, Sec. 3,
Fig. 2a/2b): loop 0 is approx-N(0,1); loop t is rho_t * x_{t-1} +
sqrt(1 - rho_t^2) * n_t, element by element, kept in fp32 across loops and
rounded to bf16 when stored.  Codebook entries are drawn from the same process
(an entry's coordinate i*Tc + m is "channel" i at loop m of a fresh token), so
they have the same marginal law and loop correlation as the vectors they code.
Queries are approx-N(0,1) in bf16.

Every number is a pure function of (seed, stream tag, layer, loop, flat index)
through Philox4x32-10, so any slice can be regenerated alone.  The fp32
arithmetic of the AR(1) recursion is fixed (multiply, multiply, add; each
rounded, no fused multiply-add) so the CUDA twin reproduces it bit for bit.

Nothing here computes anything of the quantisation method itself.
"""
from __future__ import annotations

import dataclasses
from typing import Sequence

import numpy as np

from .philox import philox4x32, approx_normal_from_words, f32_to_bf16_bits, bf16_bits_to_f32

SEED_BASE = 20261102
KEY1 = 0x4C565142          # second key word, fixed

TAG_K, TAG_V, TAG_Q, TAG_CBK, TAG_CBV, TAG_LEN, TAG_IDX, TAG_TW, TAG_TP = 1, 2, 3, 4, 5, 6, 7, 8, 9


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int
    L: int
    T: int
    Tc: int
    Hkv: int
    Hq: int
    D: int
    c: int
    K: int
    B: int
    Nmax: int
    rho: tuple            # rho[t] for t = 1..T-1 (index 0 unused, kept 0.0)
    len_lo: int = -1      # if >= 0, lengths uniform in [len_lo, Nmax]
    theta: float = 1.0e4
    ncb: int = 1          # codebooks per (layer, block, head, K|V): 1 shared, or D/c (one per channel group)
    tasq: bool = False    # keys coded after the TaSQ transform (LoopVQ paper, App. B)

    @property
    def G(self) -> int:
        return self.c * self.Tc

    @property
    def NB(self) -> int:
        return self.T // self.Tc

    @property
    def seed(self) -> int:
        return SEED_BASE + self.cfg_id

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _rho(vals: Sequence[float], T: int) -> tuple:
    if len(vals) == 1:
        vals = list(vals) * (T - 1)
    assert len(vals) == T - 1
    return (0.0,) + tuple(float(v) for v in vals)


WORKLOADS = {
    "tiny": Workload("tiny", 0, L=1, T=4, Tc=4, Hkv=1, Hq=1, D=64, c=4, K=256, B=1, Nmax=256,
                     rho=_rho((0.7, 0.8, 0.9), 4)),
    "ctx4k": Workload("ctx4k", 1, L=24, T=4, Tc=4, Hkv=16, Hq=16, D=128, c=4, K=256, B=32, Nmax=4096,
                      rho=_rho((0.7, 0.8, 0.9), 4)),
    "ctx32k": Workload("ctx32k", 2, L=24, T=4, Tc=4, Hkv=16, Hq=16, D=128, c=4, K=256, B=8, Nmax=32768,
                       rho=_rho((0.7, 0.8, 0.9), 4), len_lo=16384),
    "gqa16k": Workload("gqa16k", 3, L=24, T=4, Tc=4, Hkv=4, Hq=16, D=128, c=8, K=256, B=64, Nmax=16384,
                       rho=_rho((0.6, 0.8, 0.95), 4)),
    "deep32": Workload("deep32", 4, L=4, T=32, Tc=4, Hkv=40, Hq=40, D=128, c=4, K=256, B=2, Nmax=8192,
                       rho=_rho((0.9,), 32)),
    "ctx32k_cq": Workload("ctx32k_cq", 2, L=24, T=4, Tc=1, Hkv=16, Hq=16, D=128, c=16, K=256, B=8, Nmax=32768,
                          rho=_rho((0.7, 0.8, 0.9), 4), len_lo=16384),
    "ctx32k_pg": Workload("ctx32k_pg", 2, L=24, T=4, Tc=4, Hkv=16, Hq=16, D=128, c=4, K=256, B=8, Nmax=32768,
                          rho=_rho((0.7, 0.8, 0.9), 4), len_lo=16384, ncb=32),
    "ctx32k_tasq": Workload("ctx32k_tasq", 2, L=24, T=4, Tc=4, Hkv=16, Hq=16, D=128, c=4, K=256, B=8, Nmax=32768,
                            rho=_rho((0.7, 0.8, 0.9), 4), len_lo=16384, tasq=True),
}


def rho_sigma_f32(w: Workload):
    """Per-loop fp32 AR(1) coefficients: rho_t and sigma_t = sqrt(1 - rho_t^2) (fp64, then rounded)."""
    rho = np.array(w.rho, dtype=np.float64)
    sig = np.sqrt(1.0 - rho * rho)
    sig[0] = 1.0
    return rho.astype(np.float32), sig.astype(np.float32)


def _normal(seed, tag, layer, step, flat):
    flat = np.asarray(flat, dtype=np.uint64)
    lo = flat & np.uint64(0xFFFFFFFF)
    hi = flat >> np.uint64(32)
    ctr3 = np.uint64((tag << 24) | layer)
    w = philox4x32(lo, hi, np.uint64(step), ctr3, seed, KEY1)
    return approx_normal_from_words(*w)


def _ar1(w: Workload, tag, layer, flat, t_first: int, t_last: int, t_lo_chain: int = 0):
    """AR(1) chain over loops t_lo_chain..t_last at the given flat indices; returns fp32 [t_last-t_first+1, ...]."""
    rho, sig = rho_sigma_f32(w)
    out = []
    x = None
    for t in range(t_lo_chain, t_last + 1):
        n = _normal(w.seed, tag, layer, t, flat)
        if x is None:
            x = n
        else:
            a = (rho[t] * x).astype(np.float32)
            b = (sig[t] * n).astype(np.float32)
            x = (a + b).astype(np.float32)
        if t >= t_first:
            out.append(x)
    return np.stack(out, axis=0)


def kv_flat(w: Workload, b, tok, h, d):
    return ((np.asarray(b, np.uint64) * np.uint64(w.Nmax) + np.asarray(tok, np.uint64)) * np.uint64(w.Hkv)
            + np.asarray(h, np.uint64)) * np.uint64(w.D) + np.asarray(d, np.uint64)


def kv_loops(w: Workload, layer: int, kv: int, t_first: int, t_last: int,
             b: Sequence[int], tok: Sequence[int], h: Sequence[int], dtype: str = "bf16"):
    """Pre-RoPE K (kv=0) or V (kv=1) for loops t_first..t_last as [nt][len(b)][len(tok)][len(h)][D].

    dtype "bf16" returns uint16 bit patterns, "f32" returns the unrounded fp32 chain."""
    b = np.asarray(b, np.uint64)[:, None, None, None]
    tok = np.asarray(tok, np.uint64)[None, :, None, None]
    h = np.asarray(h, np.uint64)[None, None, :, None]
    d = np.arange(w.D, dtype=np.uint64)[None, None, None, :]
    flat = kv_flat(w, b, tok, h, d)
    x = _ar1(w, TAG_K if kv == 0 else TAG_V, layer, flat, t_first, t_last)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


def codebook(w: Workload, layer: int, block: int, kv: int, h: int, g: int = 0):
    """bf16 bits [K][G] of codebook g (0 when shared); coordinate i*Tc + m holds 'channel' i at loop m of
    entry r's fresh token.  Codebook g of head h draws from counters ((h * ncb + g) * K + r) * c + i."""
    r = np.arange(w.K, dtype=np.uint64)[:, None]
    i = np.arange(w.c, dtype=np.uint64)[None, :]
    flat = ((np.uint64(h) * np.uint64(w.ncb) + np.uint64(g)) * np.uint64(w.K) + r) * np.uint64(w.c) + i   # [K][c]
    t0 = block * w.Tc
    x = _ar1(w, TAG_CBK if kv == 0 else TAG_CBV, layer, flat, t0, t0 + w.Tc - 1, t_lo_chain=t0)  # [Tc][K][c]
    x = np.transpose(x, (1, 2, 0)).reshape(w.K, w.G)                          # [K][c*Tc], coord i*Tc+m
    return f32_to_bf16_bits(x)


def codebooks(w: Workload, layer: int, block: int, kv: int, h: int):
    """bf16 bits [ncb][K][G]: every codebook of (layer, block, K|V, head)."""
    return np.stack([codebook(w, layer, block, kv, h, g) for g in range(w.ncb)])


def queries(w: Workload, layer: int, t: int, b: Sequence[int] = None, hq: Sequence[int] = None,
            gain: float = 1.0):
    """bf16 bits [len(b)][len(hq)][D]; the query is taken as already rotated at its own position."""
    b = np.arange(w.B) if b is None else np.asarray(b)
    hq = np.arange(w.Hq) if hq is None else np.asarray(hq)
    flat = ((b.astype(np.uint64)[:, None, None] * np.uint64(w.Hq) + hq.astype(np.uint64)[None, :, None])
            * np.uint64(w.D) + np.arange(w.D, dtype=np.uint64)[None, None, :])
    x = _normal(w.seed, TAG_Q, layer, t, flat)
    if gain != 1.0:
        x = (x * np.float32(gain)).astype(np.float32)
    return f32_to_bf16_bits(x)


def lengths(w: Workload) -> np.ndarray:
    """int32 [B]: all Nmax, or uniform in [len_lo, Nmax] drawn per sequence."""
    if w.len_lo < 0:
        return np.full(w.B, w.Nmax, dtype=np.int32)
    b = np.arange(w.B, dtype=np.uint64)
    w0, _, _, _ = philox4x32(b, 0, 0, np.uint64(TAG_LEN << 24), w.seed, KEY1)
    span = w.Nmax - w.len_lo + 1
    return (w.len_lo + (w0.astype(np.int64) % span)).astype(np.int32)


def tasq_weights(w: Workload) -> np.ndarray:
    """TaSQ channel weights fp32 [L][T][Hkv][D]: exp(0.25 n) for the low channel of each RoPE pair,
    the same weight for its partner (a stand-in for calibrated query moments, which need a model)."""
    L, T, H, h2 = w.L, w.T, w.Hkv, w.D // 2
    out = np.empty((L, T, H, w.D), np.float32)
    flat = np.arange(H * h2, dtype=np.uint64)
    for layer in range(L):
        for t in range(T):
            n = _normal(w.seed, TAG_TW, layer, t, flat).reshape(H, h2)
            half = np.exp(np.float32(0.25) * n.astype(np.float32)).astype(np.float32)
            out[layer, t] = np.concatenate([half, half], axis=1)
    return out


def tasq_perm(w: Workload) -> np.ndarray:
    """TaSQ low-channel orders int16 [L][NB][Hkv][D/2]: a seeded permutation per (layer, block, head)
    (a stand-in for the covariance grouping, which needs real caches)."""
    L, NB, H, h2 = w.L, w.NB, w.Hkv, w.D // 2
    out = np.empty((L, NB, H, h2), np.int16)
    for layer in range(L):
        for blk in range(NB):
            flat = np.arange(H * h2, dtype=np.uint64)
            k0, _, _, _ = philox4x32(flat & np.uint64(0xFFFFFFFF), flat >> np.uint64(32), np.uint64(blk),
                                     np.uint64((TAG_TP << 24) | layer), w.seed, KEY1)
            keys = k0.reshape(H, h2).astype(np.uint64) * np.uint64(h2) + np.arange(h2, dtype=np.uint64)[None, :]
            out[layer, blk] = np.argsort(keys, axis=1).astype(np.int16)
    return out


def random_indices(w: Workload, layer: int, block: int, kv: int, b: int, h: int, tok: Sequence[int]):
    """uint8 [len(tok)][D/c] code indices drawn uniformly in [0, K): decode input independent of any encoder."""
    ng = w.D // w.c
    tok = np.asarray(tok, np.uint64)[:, None]
    gi = np.arange(ng, dtype=np.uint64)[None, :]
    flat = ((np.uint64(b) * np.uint64(w.Hkv) + np.uint64(h)) * np.uint64(w.Nmax) + tok) * np.uint64(ng) + gi
    w0, _, _, _ = philox4x32(flat & np.uint64(0xFFFFFFFF), flat >> np.uint64(32),
                             np.uint64(block * 2 + kv), np.uint64((TAG_IDX << 24) | layer), w.seed, KEY1)
    return (w0 % np.uint32(w.K)).astype(np.uint8)


__all__ = ["Workload", "WORKLOADS", "kv_loops", "codebook", "codebooks", "tasq_weights", "tasq_perm", "queries", "lengths", "random_indices",
           "rho_sigma_f32", "bf16_bits_to_f32", "f32_to_bf16_bits"]
