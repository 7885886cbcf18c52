"""ctypes front end of the CPU checker (test infrastructure only).

Thin marshalling over ``libloopvq_oracle.so``; every computation happens in
``loopvq_oracle.c``, whose header cites the passages each function follows.
bf16 inputs are widened here to the exactly equal fp32 values.
"""
from __future__ import annotations

import ctypes as C
import math

import numpy as np

from .build import build

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        I, D_ = C.c_int, C.c_double
        _lib.ora_encode.argtypes = [f32p, I, I, I, I, f32p, I, u8p]
        _lib.ora_encode.restype = None
        _lib.ora_dist64.argtypes = [f32p, I, I, I, I, f32p, I, I, I]
        _lib.ora_dist64.restype = D_
        _lib.ora_dequant.argtypes = [u8p, I, I, I, I, I, f32p, f64p]
        _lib.ora_dequant.restype = None
        _lib.ora_rope.argtypes = [f64p, I, I, D_, I]
        _lib.ora_rope.restype = None
        _lib.ora_attention.argtypes = [f64p, f64p, f64p, I, I, D_, f64p, C.POINTER(D_)]
        _lib.ora_attention.restype = None
        _lib.ora_attention_splits.argtypes = [f64p, f64p, f64p, I, I, D_, i32p, I, f64p, C.POINTER(D_)]
        _lib.ora_attention_splits.restype = None
        _lib.ora_decode.argtypes = [f64p, u8p, u8p, f32p, f32p, I, I, I, I, I, D_, D_, f64p, C.POINTER(D_)]
        _lib.ora_decode.restype = None
        _lib.ora_decode_windowed.argtypes = [f64p, f64p, f64p, I, u8p, u8p, f32p, f32p, I, I, I, I, I, I, D_, D_,
                                             f64p, C.POINTER(D_)]
        _lib.ora_decode_windowed.restype = None
        _lib.ora_encode_pg.argtypes = [f32p, I, I, I, I, f32p, I, u8p]
        _lib.ora_encode_pg.restype = None
        _lib.ora_dist64_pg.argtypes = [f32p, I, I, I, I, f32p, I, I, I, I]
        _lib.ora_dist64_pg.restype = D_
        _lib.ora_dequant_pg.argtypes = [u8p, I, I, I, I, I, f32p, I, f64p]
        _lib.ora_dequant_pg.restype = None
        _lib.ora_decode_pg.argtypes = [f64p, u8p, u8p, f32p, f32p, I, I, I, I, I, I, D_, D_, f64p, C.POINTER(D_)]
        _lib.ora_decode_pg.restype = None
        i16p = np.ctypeslib.ndpointer(np.int16, flags="C_CONTIGUOUS")
        _lib.ora_round_fp16.argtypes = [D_]
        _lib.ora_round_fp16.restype = D_
        _lib.ora_tasq_sigma.argtypes = [f32p, f32p, I, I, I, f64p]
        _lib.ora_tasq_sigma.restype = None
        _lib.ora_tasq_transform.argtypes = [f32p, f32p, f64p, I, I, f32p]
        _lib.ora_tasq_transform.restype = None
        _lib.ora_tasq_encode.argtypes = [f32p, f32p, f64p, i16p, I, I, I, I, f32p, I, u8p]
        _lib.ora_tasq_encode.restype = None
        _lib.ora_tasq_dequant.argtypes = [u8p, I, I, I, I, I, f32p, i16p, f32p, f64p, f64p]
        _lib.ora_tasq_dequant.restype = None
        _lib.ora_tasq_decode.argtypes = [f64p, u8p, u8p, f32p, f32p, i16p, f32p, f64p, I, I, I, I, I, D_, D_, f64p,
                                         C.POINTER(D_)]
        _lib.ora_tasq_decode.restype = None
    return _lib


def widen_bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the equal fp32 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def encode(x, E, c: int) -> np.ndarray:
    """x fp32 [Tc][N][D] (one block), E fp32 [K][G] -> uint8 [N][D/c]."""
    x = _f32(x)
    E = _f32(E)
    Tc, N, D = x.shape
    K, G = E.shape
    assert G == c * Tc and D % c == 0 and K <= 256
    out = np.zeros((N, D // c), dtype=np.uint8)
    lib().ora_encode(x, Tc, N, D, c, E, K, out)
    return out


def dist64(x, E, c: int, n: int, g: int, r: int) -> float:
    x = _f32(x)
    E = _f32(E)
    Tc, N, D = x.shape
    return lib().ora_dist64(x, Tc, N, D, c, E, n, g, r)


def dequant(idx, E, c: int, Tc: int, m: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    E = _f32(E)
    N, ng = idx.shape
    D = ng * c
    out = np.zeros((N, D), dtype=np.float64)
    lib().ora_dequant(idx, N, D, c, Tc, m, E, out)
    return out


def rope(x, theta: float = 1.0e4, pos0: int = 0) -> np.ndarray:
    y = np.array(x, dtype=np.float64, order="C", copy=True)
    N, D = y.shape
    lib().ora_rope(y, N, D, theta, pos0)
    return y


def attention(q, k, v, scale: float):
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    N, D = k.shape if k.size else (0, q.shape[0])
    out = np.zeros(D, dtype=np.float64)
    lse = C.c_double(0.0)
    lib().ora_attention(q, k.reshape(-1, D) if N else np.zeros((1, D)), v.reshape(-1, D) if N else np.zeros((1, D)),
                        N, D, scale, out, C.byref(lse))
    return out, lse.value


def attention_splits(q, k, v, scale: float, bounds):
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    N, D = k.shape
    b = np.ascontiguousarray(bounds, dtype=np.int32)
    out = np.zeros(D, dtype=np.float64)
    lse = C.c_double(0.0)
    lib().ora_attention_splits(q, k, v, N, D, scale, b, len(b) - 1, out, C.byref(lse))
    return out, lse.value


def decode(q, idx_k, idx_v, E_k, E_v, c: int, Tc: int, m: int, theta: float = 1.0e4, scale: float = None):
    """One query over a coded cache of N = len(idx_k) tokens at loop step m of the block."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    D = q.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    idx_k = np.ascontiguousarray(idx_k, dtype=np.uint8).reshape(-1, D // c)
    idx_v = np.ascontiguousarray(idx_v, dtype=np.uint8).reshape(-1, D // c)
    N = idx_k.shape[0]
    out = np.zeros(D, dtype=np.float64)
    lse = C.c_double(0.0)
    lib().ora_decode(q, idx_k if N else np.zeros((1, D // c), np.uint8), idx_v if N else np.zeros((1, D // c), np.uint8),
                     _f32(E_k), _f32(E_v), N, D, c, Tc, m, theta, scale, out, C.byref(lse))
    return out, lse.value


def decode_windowed(q, k_win, v_win, idx_k, idx_v, E_k, E_v, c: int, Tc: int, m: int, lo: int,
                    theta: float = 1.0e4, scale: float = None):
    """One query over NW bf16 window tokens (k_win already rotated, v_win: [NW][D]) and the coded
    tokens lo .. lo + len(idx_k) - 1 (codes idx_k / idx_v [n][D/c]) at loop step m of the block."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    D = q.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    kw = np.ascontiguousarray(k_win, dtype=np.float64).reshape(-1, D)
    vw = np.ascontiguousarray(v_win, dtype=np.float64).reshape(-1, D)
    idx_k = np.ascontiguousarray(idx_k, dtype=np.uint8).reshape(-1, D // c)
    idx_v = np.ascontiguousarray(idx_v, dtype=np.uint8).reshape(-1, D // c)
    NW, NC = kw.shape[0], idx_k.shape[0]
    out = np.zeros(D, dtype=np.float64)
    lse = C.c_double(0.0)
    z64 = np.zeros((1, D), np.float64)
    z8 = np.zeros((1, D // c), np.uint8)
    lib().ora_decode_windowed(q, kw if NW else z64, vw if NW else z64, NW, idx_k if NC else z8, idx_v if NC else z8,
                              _f32(E_k), _f32(E_v), lo, lo + NC, D, c, Tc, m, theta, scale, out, C.byref(lse))
    return out, lse.value


# ---- one codebook per channel group: E is [D/c][K][G]

def encode_pg(x, E, c: int) -> np.ndarray:
    x = _f32(x)
    Tc, N, D = x.shape
    E = _f32(E)
    ng, K, G = E.shape
    assert ng == D // c and G == c * Tc
    idx = np.zeros((N, ng), dtype=np.uint8)
    if N:
        lib().ora_encode_pg(x, Tc, N, D, c, E, K, idx)
    return idx


def dist64_pg(x, E, c: int, n: int, g: int, r: int) -> float:
    x = _f32(x)
    Tc, N, D = x.shape
    E = _f32(E)
    return lib().ora_dist64_pg(x, Tc, N, D, c, E, E.shape[1], n, g, r)


def dequant_pg(idx, E, c: int, Tc: int, m: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    E = _f32(E)
    N = idx.shape[0]
    D = idx.shape[1] * c
    out = np.zeros((N, D), dtype=np.float64)
    if N:
        lib().ora_dequant_pg(idx, N, D, c, Tc, m, E, E.shape[1], out)
    return out


def decode_pg(q, idx_k, idx_v, E_k, E_v, c: int, Tc: int, m: int, theta: float = 1.0e4, scale: float = None):
    """decode() with per-group codebooks E_k, E_v: [D/c][K][G]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    D = q.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    idx_k = np.ascontiguousarray(idx_k, dtype=np.uint8).reshape(-1, D // c)
    idx_v = np.ascontiguousarray(idx_v, dtype=np.uint8).reshape(-1, D // c)
    N = idx_k.shape[0]
    E_k, E_v = _f32(E_k), _f32(E_v)
    out = np.zeros(D, dtype=np.float64)
    lse = C.c_double(0.0)
    z8 = np.zeros((1, D // c), np.uint8)
    lib().ora_decode_pg(q, idx_k if N else z8, idx_v if N else z8, E_k, E_v, E_k.shape[1], N, D, c, Tc, m, theta,
                        scale, out, C.byref(lse))
    return out, lse.value


# ---- TaSQ before loop-axis coupling (App. B)

def round_fp16(x: float) -> float:
    return lib().ora_round_fp16(float(x))


def tasq_sigma(k, w) -> np.ndarray:
    """k: [Hkv][N][D] keys of one (loop step, layer, sequence), w: [Hkv][D] -> sigma [N] (fp16 values)."""
    k, w = _f32(k), _f32(w)
    Hkv, N, D = k.shape
    out = np.zeros(N, dtype=np.float64)
    if N:
        lib().ora_tasq_sigma(k, w, Hkv, N, D, out)
    return out


def tasq_transform(k, w, sigma) -> np.ndarray:
    """k: [N][D], w: [D], sigma: [N] -> u [N][D] fp32."""
    k, w = _f32(k), _f32(w)
    N, D = k.shape
    u = np.zeros((N, D), dtype=np.float32)
    if N:
        lib().ora_tasq_transform(k, w, np.ascontiguousarray(sigma, np.float64), N, D, u)
    return u


def tasq_encode(x, w, sigma, perm, E, c: int) -> np.ndarray:
    """x: [Tc][N][D] keys of one (layer, block, head), w: [Tc][D], sigma: [Tc][N], perm: [D/2]."""
    x = _f32(x)
    Tc, N, D = x.shape
    E = _f32(E)
    idx = np.zeros((N, D // c), dtype=np.uint8)
    if N:
        lib().ora_tasq_encode(x, _f32(w), np.ascontiguousarray(sigma, np.float64),
                              np.ascontiguousarray(perm, np.int16), Tc, N, D, c, E, E.shape[0], idx)
    return idx


def tasq_dequant(idx, E, c: int, Tc: int, m: int, perm, w, sigma) -> np.ndarray:
    """Keys of loop step m rebuilt with the transform inverted; w: [D] and sigma: [N] of that step."""
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    N = idx.shape[0]
    D = idx.shape[1] * c
    out = np.zeros((N, D), dtype=np.float64)
    if N:
        lib().ora_tasq_dequant(idx, N, D, c, Tc, m, _f32(E), np.ascontiguousarray(perm, np.int16), _f32(w),
                               np.ascontiguousarray(sigma, np.float64), out)
    return out


def tasq_decode(q, idx_k, idx_v, E_k, E_v, perm, w, sigma, c: int, Tc: int, m: int, theta: float = 1.0e4,
                scale: float = None):
    q = np.ascontiguousarray(q, dtype=np.float64)
    D = q.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    idx_k = np.ascontiguousarray(idx_k, dtype=np.uint8).reshape(-1, D // c)
    idx_v = np.ascontiguousarray(idx_v, dtype=np.uint8).reshape(-1, D // c)
    N = idx_k.shape[0]
    out = np.zeros(D, dtype=np.float64)
    lse = C.c_double(0.0)
    z8 = np.zeros((1, D // c), np.uint8)
    sig = np.ascontiguousarray(sigma, np.float64) if N else np.ones(1)
    lib().ora_tasq_decode(q, idx_k if N else z8, idx_v if N else z8, _f32(E_k), _f32(E_v),
                          np.ascontiguousarray(perm, np.int16), _f32(w), sig, N, D, c, Tc, m, theta, scale, out,
                          C.byref(lse))
    return out, lse.value
