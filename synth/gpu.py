"""Device-side bulk generation of the synthetic workloads (same numbers as synth.workloads)."""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

from .philox import IH_SCALE
from .workloads import (Workload, rho_sigma_f32, TAG_K, TAG_V, TAG_Q, TAG_CBK, TAG_CBV, TAG_IDX)

_LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libloopvq_synth.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB):
            raise RuntimeError(f"{_LIB} missing: build with synth/build.py")
        L = C.CDLL(_LIB)
        u32, i, f, vp, sz = C.c_uint32, C.c_int, C.c_float, C.c_void_p, C.c_size_t
        fp = C.POINTER(C.c_float)
        L.synth_kv.argtypes = [vp, u32, u32, i, i, i, i, i, i, fp, fp, f, vp]
        L.synth_q.argtypes = [vp, u32, u32, i, sz, f, f, vp]
        L.synth_codebook.argtypes = [vp, u32, i, i, i, i, i, i, i, fp, fp, f, u32, u32, vp]
        L.synth_idx.argtypes = [vp, u32, u32, i, i, i, i, i, i, vp]
        for n in ("synth_kv", "synth_q", "synth_codebook", "synth_idx"):
            getattr(L, n).restype = i
        _lib = L
    return _lib


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _coef(w: Workload):
    rho, sig = rho_sigma_f32(w)
    return (np.ascontiguousarray(rho, np.float32), np.ascontiguousarray(sig, np.float32))


def _fp(a):
    return a.ctypes.data_as(C.POINTER(C.c_float))


def _ok(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def fill_kv(w: Workload, layer: int, kv: int, t_first: int, t_last: int, out: torch.Tensor, B: int = None,
            Nmax: int = None):
    """out: bf16 [t_last-t_first+1][B][Nmax][Hkv][D] on the device."""
    B = w.B if B is None else B
    Nmax = w.Nmax if Nmax is None else Nmax
    assert out.dtype == torch.bfloat16 and out.is_contiguous()
    assert out.numel() == (t_last - t_first + 1) * B * Nmax * w.Hkv * w.D
    rho, sig = _coef(w)
    tagl = ((TAG_K if kv == 0 else TAG_V) << 24) | layer
    _ok(lib().synth_kv(out.data_ptr(), w.seed, tagl, t_first, t_last, B, Nmax, w.Hkv, w.D, _fp(rho), _fp(sig),
                       float(IH_SCALE), _stream()), "synth_kv")


def fill_q(w: Workload, layer: int, t: int, out: torch.Tensor, gain: float = 1.0):
    assert out.dtype == torch.bfloat16 and out.is_contiguous() and out.numel() == w.B * w.Hq * w.D
    _ok(lib().synth_q(out.data_ptr(), w.seed, (TAG_Q << 24) | layer, t, out.numel(), float(IH_SCALE), float(gain),
                      _stream()), "synth_q")


def fill_codebook(w: Workload, out: torch.Tensor):
    """out: the cache codebook buffer [L][NB][2][Hkv][NCB][K][G] (bf16 bits)."""
    rho, sig = _coef(w)
    _ok(lib().synth_codebook(out.data_ptr(), w.seed, w.L, w.NB, w.Tc, w.Hkv, w.ncb, w.K, w.c, _fp(rho), _fp(sig),
                             float(IH_SCALE), TAG_CBK, TAG_CBV, _stream()), "synth_codebook")


def fill_idx(w: Workload, layer: int, block: int, out_words: torch.Tensor, B: int = None):
    """Uniform codes for one (layer, block) run of index words [B][Hkv][Nmax/4][NP][4]."""
    B = w.B if B is None else B
    NP = w.D // (2 * w.c)
    assert out_words.numel() == B * w.Hkv * w.Nmax * NP
    _ok(lib().synth_idx(out_words.data_ptr(), w.seed, (TAG_IDX << 24) | layer, block, B, w.Hkv, w.Nmax, NP, w.K,
                        _stream()), "synth_idx")
