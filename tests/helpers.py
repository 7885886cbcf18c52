"""Test-side helpers: the documented index-word layout of include/loopvq.h and cache set-up.

Nothing here computes the method; it only moves bytes between the checker's
natural arrays ([N][D/c] codes per K|V) and the library's packed words.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from synth import codebooks, Workload, codebook, kv_loops, queries, lengths, bf16_bits_to_f32


def pack_words(idx_k: np.ndarray, idx_v: np.ndarray, NP: int) -> np.ndarray:
    """[N][2NP] K and V codes -> uint32 words in tile order [N/4][NP][4] (N multiple of 4)."""
    N = idx_k.shape[0]
    k = idx_k.astype(np.uint32)
    v = idx_v.astype(np.uint32)
    w = k[:, :NP] | (k[:, NP:] << 8) | (v[:, :NP] << 16) | (v[:, NP:] << 24)      # [N][NP]
    return np.ascontiguousarray(w.reshape(N // 4, 4, NP).transpose(0, 2, 1)).reshape(-1)


def unpack_words(words: np.ndarray, N: int, NP: int):
    w = words.reshape(N // 4, NP, 4).transpose(0, 2, 1).reshape(N, NP).astype(np.uint32)
    k = np.concatenate([w & 0xFF, (w >> 8) & 0xFF], axis=1).astype(np.uint8)
    v = np.concatenate([(w >> 16) & 0xFF, (w >> 24) & 0xFF], axis=1).astype(np.uint8)
    return k, v


def words_view(cache, layer: int, block: int, b: int, h: int) -> torch.Tensor:
    """The (layer, block, b, h) run of the device index buffer."""
    per = cache.Nmax * cache.NP
    base = (((layer * cache.NB + block) * cache.B + b) * cache.Hkv + h) * per
    return cache.idx[base:base + per]


def codebook_view(cache, layer: int, block: int, kv: int, h: int) -> torch.Tensor:
    """The codebook(s) of (layer, block, K|V, head): [NCB * K * G] elements, NCB = 1 when shared."""
    G = cache.c * cache.Tc
    n = cache.ncb * cache.K * G
    base = (((layer * cache.NB + block) * 2 + kv) * cache.Hkv + h) * n
    return cache.codebook[base:base + n]


def make_cache(w: Workload, device="cuda", codebooks="numpy"):
    """Cache with the workload's shapes, numpy-generated codebooks uploaded, prepared."""
    import looped_lm_decode_b200 as LQ
    cache = LQ.Cache(w.L, w.T, w.Tc, w.Hkv, w.Hq, w.D, w.c, w.K, w.B, w.Nmax, w.theta, device=device, ncb=w.ncb)
    if codebooks == "numpy":
        for layer in range(w.L):
            for blk in range(w.NB):
                for kv in range(2):
                    for h in range(w.Hkv):
                        cb = np_codebook_bits(w, layer, blk, kv, h).view(np.int16).reshape(-1)
                        codebook_view(cache, layer, blk, kv, h).copy_(torch.from_numpy(cb))
    else:
        from synth import gpu as SG
        SG.fill_codebook(w, cache.codebook)
    LQ.prepare(cache)
    return cache


def np_codebook_bits(w: Workload, layer, block, kv, h):
    """[K][G] bits when the codebook is shared, [NCB][K][G] with one per channel group."""
    return codebook(w, layer, block, kv, h) if w.ncb == 1 else codebooks(w, layer, block, kv, h)


def np_codebook_f32(w: Workload, layer, block, kv, h):
    return bf16_bits_to_f32(np_codebook_bits(w, layer, block, kv, h))


def attn_tolerance_ok(out, ref, lse=None, lse_ref=None, rel=2e-3, lse_tol=1e-3):
    """max|out - ref| <= rel * ||ref||_inf over the call tensor; |lse - lse_ref| <= lse_tol."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    err = np.abs(out - ref).max()
    ok = err <= rel * scale if scale > 0 else err == 0
    msg = f"max|err|={err:.3e} bound={rel * scale:.3e}"
    if lse is not None:
        fin = np.isfinite(lse_ref)
        ok = ok and np.array_equal(np.isfinite(lse), fin)
        if fin.any():
            le = np.abs(np.asarray(lse)[fin] - np.asarray(lse_ref)[fin]).max()
            ok = ok and le <= lse_tol
            msg += f" lse_err={le:.3e}"
    return ok, msg
