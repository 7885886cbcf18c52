"""Python binding of libloopvq (the C ABI in include/loopvq.h).

Argument marshalling only: torch provides device memory and streams, and
every step of the path runs in the library's CUDA kernels.  Loading fails
loudly if the library has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libloopvq.so")

(LOOPVQ_OK, LOOPVQ_ERR_INVALID_ARG, LOOPVQ_ERR_UNSUPPORTED, LOOPVQ_ERR_WORKSPACE, LOOPVQ_ERR_CUDA, LOOPVQ_ERR_TIMEOUT,
 LOOPVQ_ERR_OVERFLOW) = range(7)
LOOPVQ_BF16, LOOPVQ_FP32 = 0, 1

EXPORTS = ("loopvq_idx_words", "loopvq_codebook_elems", "loopvq_slice_elems", "loopvq_rope_elems",
           "loopvq_prepare", "loopvq_encode", "loopvq_decode_workspace_bytes", "loopvq_decode_attn",
           "loopvq_dequant_debug", "loopvq_last_error", "loopvq_abi_version",
           "loopvq_decode_attn_noalloc", "loopvq_noalloc_scratch_bytes", "loopvq_decode_attn_range",
           "loopvq_bf16_decode_workspace_bytes", "loopvq_bf16_decode_attn", "loopvq_merge2",
           "loopvq_window_slots", "loopvq_window_advance", "loopvq_window_append",
           "loopvq_window_workspace_bytes", "loopvq_window_decode_attn", "loopvq_window_append_decode_attn",
           "loopvq_tasq_w_elems",
           "loopvq_tasq_perm_elems", "loopvq_tasq_sigma_elems", "loopvq_tasq_encode", "loopvq_tasq_decode_attn",
           "loopvq_fault_check", "loopvq_set_wait_limit_ns", "loopvq_wait_limit_ns")


class CacheDesc(C.Structure):
    """Mirror of struct loopvq_cache."""
    _fields_ = [("L", C.c_int32), ("T", C.c_int32), ("Tc", C.c_int32), ("Hkv", C.c_int32),
                ("Hq", C.c_int32), ("D", C.c_int32), ("c", C.c_int32), ("K", C.c_int32),
                ("B", C.c_int32), ("Nmax", C.c_int32), ("theta", C.c_float),
                ("idx", C.c_void_p), ("codebook", C.c_void_p), ("slices", C.c_void_p), ("rope", C.c_void_p),
                ("ncb", C.c_int32)]


class Bf16CacheDesc(C.Structure):
    """Mirror of struct loopvq_bf16_cache."""
    _fields_ = [("B", C.c_int32), ("Hkv", C.c_int32), ("Hq", C.c_int32), ("D", C.c_int32), ("Nmax", C.c_int32),
                ("k", C.c_void_p), ("v", C.c_void_p)]


class WindowDesc(C.Structure):
    """Mirror of struct loopvq_window."""
    _fields_ = [("L", C.c_int32), ("T", C.c_int32), ("B", C.c_int32), ("Hkv", C.c_int32), ("Hq", C.c_int32),
                ("D", C.c_int32), ("n_sink", C.c_int32), ("n_recent", C.c_int32), ("k_rot", C.c_void_p),
                ("k_pre", C.c_void_p), ("v", C.c_void_p), ("fill", C.c_void_p), ("coded_end", C.c_void_p)]


class TasqDesc(C.Structure):
    """Mirror of struct loopvq_tasq."""
    _fields_ = [("w", C.c_void_p), ("perm", C.c_void_p), ("sigma", C.c_void_p)]


class LoopVQError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"loopvq status {status}: {msg}")
        self.status = status


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with looped_lm_decode_b200/build.py "
                               "(nvcc, sm_100a); there is no CPU fallback")
        L = C.CDLL(LIB_PATH)
        P = C.POINTER(CacheDesc)
        vp, i, sz, f = C.c_void_p, C.c_int, C.c_size_t, C.c_float
        for name in ("loopvq_idx_words", "loopvq_codebook_elems", "loopvq_slice_elems", "loopvq_rope_elems"):
            getattr(L, name).argtypes = [P]
            getattr(L, name).restype = sz
        L.loopvq_prepare.argtypes = [P, vp]
        L.loopvq_encode.argtypes = [P, i, i, vp, vp, i, C.POINTER(C.c_int64), i, i, i, i, vp]
        L.loopvq_decode_workspace_bytes.argtypes = [P, i]
        L.loopvq_decode_workspace_bytes.restype = sz
        L.loopvq_decode_attn.argtypes = [P, i, i, vp, vp, i, f, vp, vp, vp, sz, vp]
        L.loopvq_dequant_debug.argtypes = [P, i, i, i, i, i, i, i, vp, vp]
        L.loopvq_decode_attn_noalloc.argtypes = [P, i, i, vp, vp, i, f, vp, vp, vp]
        L.loopvq_decode_attn_noalloc.restype = i
        L.loopvq_decode_attn_range.argtypes = [P, i, i, vp, vp, vp, i, f, vp, vp, vp, sz, vp]
        L.loopvq_decode_attn_range.restype = i
        PB = C.POINTER(Bf16CacheDesc)
        L.loopvq_bf16_decode_workspace_bytes.argtypes = [PB, i]
        L.loopvq_bf16_decode_workspace_bytes.restype = sz
        L.loopvq_bf16_decode_attn.argtypes = [PB, vp, vp, vp, i, f, vp, vp, vp, sz, vp]
        L.loopvq_bf16_decode_attn.restype = i
        L.loopvq_merge2.argtypes = [vp, vp, vp, vp, i, i, vp, vp, vp]
        L.loopvq_merge2.restype = i
        PW = C.POINTER(WindowDesc)
        L.loopvq_window_slots.argtypes = [PW]
        L.loopvq_window_slots.restype = i
        L.loopvq_window_advance.argtypes = [PW, P, vp]
        L.loopvq_window_advance.restype = i
        L.loopvq_window_append.argtypes = [PW, i, i, vp, vp, vp, vp]
        L.loopvq_window_append.restype = i
        L.loopvq_window_workspace_bytes.argtypes = [PW, P, i]
        L.loopvq_window_workspace_bytes.restype = sz
        L.loopvq_window_decode_attn.argtypes = [PW, P, i, i, vp, i, f, vp, vp, vp, sz, vp]
        L.loopvq_window_decode_attn.restype = i
        L.loopvq_window_append_decode_attn.argtypes = [PW, P, i, i, vp, vp, vp, vp, i, f, vp, vp, vp, sz, vp]
        L.loopvq_window_append_decode_attn.restype = i
        PT = C.POINTER(TasqDesc)
        for name in ("loopvq_tasq_w_elems", "loopvq_tasq_perm_elems", "loopvq_tasq_sigma_elems"):
            getattr(L, name).argtypes = [P]
            getattr(L, name).restype = sz
        L.loopvq_tasq_encode.argtypes = [P, PT, i, i, vp, vp, i, C.POINTER(C.c_int64), i, i, i, i, vp]
        L.loopvq_tasq_encode.restype = i
        L.loopvq_tasq_decode_attn.argtypes = [P, PT, i, i, vp, vp, i, f, vp, vp, vp, sz, vp]
        L.loopvq_tasq_decode_attn.restype = i
        L.loopvq_noalloc_scratch_bytes.argtypes = []
        L.loopvq_noalloc_scratch_bytes.restype = sz
        for name in ("loopvq_prepare", "loopvq_encode", "loopvq_decode_attn", "loopvq_dequant_debug"):
            getattr(L, name).restype = i
        L.loopvq_last_error.argtypes = []
        L.loopvq_last_error.restype = C.c_char_p
        L.loopvq_abi_version.restype = i
        L.loopvq_fault_check.argtypes = [vp]
        L.loopvq_fault_check.restype = i
        L.loopvq_set_wait_limit_ns.argtypes = [C.c_uint64]
        L.loopvq_set_wait_limit_ns.restype = None
        L.loopvq_wait_limit_ns.argtypes = []
        L.loopvq_wait_limit_ns.restype = C.c_uint64
        _lib = L
    return _lib


def _check(status):
    if status != LOOPVQ_OK:
        raise LoopVQError(status, lib().loopvq_last_error().decode())


def fault_check(stream=None):
    """loopvq_fault_check: synchronise the stream, then raise LoopVQError if a kernel on this GPU recorded a
    fault (an encode wait that ran out, a window roll without room) since the last check."""
    _check(lib().loopvq_fault_check(_stream(stream)))


def set_wait_limit_ns(ns: int):
    """loopvq_set_wait_limit_ns: bound on each wait of the tensor-core encoder (process-wide)."""
    lib().loopvq_set_wait_limit_ns(int(ns))


def wait_limit_ns() -> int:
    return int(lib().loopvq_wait_limit_ns())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


class Cache:
    """Shape plus the four device buffers of a coded cache (see include/loopvq.h)."""

    def __init__(self, L, T, Tc, Hkv, Hq, D, c, K, B, Nmax, theta=1.0e4, device="cuda", alloc=True, ncb=1):
        """ncb: 1 for one codebook per (layer, block, head, K|V), D // c for one per channel group."""
        self.desc = CacheDesc(L, T, Tc, Hkv, Hq, D, c, K, B, Nmax, theta, None, None, None, None, ncb)
        self.L, self.T, self.Tc, self.Hkv, self.Hq, self.D, self.c, self.K = L, T, Tc, Hkv, Hq, D, c, K
        self.ncb = ncb
        self.B, self.Nmax, self.theta = B, Nmax, theta
        self.idx = self.codebook = self.slices = self.rope = None
        if alloc:
            n_idx = lib().loopvq_idx_words(C.byref(self.desc))
            if n_idx == 0:
                raise LoopVQError(LOOPVQ_ERR_INVALID_ARG, "invalid or unsupported cache shape")
            self.idx = torch.zeros(n_idx, dtype=torch.int32, device=device)
            self.codebook = torch.zeros(lib().loopvq_codebook_elems(C.byref(self.desc)), dtype=torch.int16, device=device)
            self.slices = torch.zeros(lib().loopvq_slice_elems(C.byref(self.desc)), dtype=torch.int16, device=device)
            self.rope = torch.zeros(lib().loopvq_rope_elems(C.byref(self.desc)), dtype=torch.float32, device=device)
            self._sync_desc()

    def _sync_desc(self):
        self.desc.idx = self.idx.data_ptr() if self.idx is not None else None
        self.desc.codebook = self.codebook.data_ptr() if self.codebook is not None else None
        self.desc.slices = self.slices.data_ptr() if self.slices is not None else None
        self.desc.rope = self.rope.data_ptr() if self.rope is not None else None

    @property
    def NB(self):
        return self.T // self.Tc

    @property
    def NP(self):
        return self.D // (2 * self.c)

    def ref(self):
        self._sync_desc()
        return C.byref(self.desc)


def prepare(cache: Cache, stream=None):
    _check(lib().loopvq_prepare(cache.ref(), _stream(stream)))


def encode(cache: Cache, layer: int, block: int, xk: torch.Tensor, xv: torch.Tensor, b0: int = 0, tok0: int = 0,
           stream=None):
    """xk, xv: [Tc][nb][ntok][Hkv][D] (bf16 or fp32, innermost dim contiguous, same strides)."""
    assert xk.shape == xv.shape and xk.stride() == xv.stride() and xk.dtype == xv.dtype
    Tc, nb, ntok, Hkv, D = xk.shape
    assert xk.stride(4) == 1
    dt = {torch.bfloat16: LOOPVQ_BF16, torch.float32: LOOPVQ_FP32}[xk.dtype]
    strides = (C.c_int64 * 4)(*xk.stride()[:4])
    _check(lib().loopvq_encode(cache.ref(), layer, block, _ptr(xk), _ptr(xv), dt, strides, b0, nb, tok0, ntok,
                               _stream(stream)))


def decode_workspace_bytes(cache: Cache, max_len: int) -> int:
    return lib().loopvq_decode_workspace_bytes(cache.ref(), max_len)


def decode_attn(cache: Cache, layer: int, t: int, q: torch.Tensor, lens: torch.Tensor, max_len: int,
                scale: float = 0.0, out=None, lse=None, workspace=None, stream=None):
    """q bf16 [B][Hq][D] (post-RoPE), lens int32 [B]; returns (out fp32 [B][Hq][D], lse fp32 [B][Hq])."""
    B, Hq, D = cache.B, cache.Hq, cache.D
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    need = decode_workspace_bytes(cache, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().loopvq_decode_attn(cache.ref(), layer, t, _ptr(q), _ptr(lens), max_len, scale, _ptr(out),
                                    _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)))
    return out, lse


def decode_attn_noalloc(cache: Cache, layer: int, t: int, q: torch.Tensor, lens: torch.Tensor, max_len: int,
                        scale: float = 0.0, out=None, lse=None, stream=None):
    """decode_attn with the library's built-in scratch array instead of a caller workspace."""
    B, Hq, D = cache.B, cache.Hq, cache.D
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check(lib().loopvq_decode_attn_noalloc(cache.ref(), layer, t, _ptr(q), _ptr(lens), max_len, scale, _ptr(out),
                                            _ptr(lse), _stream(stream)))
    return out, lse


def decode_attn_range(cache: Cache, layer: int, t: int, q: torch.Tensor, starts, lens: torch.Tensor,
                      max_len: int, scale: float = 0.0, out=None, lse=None, workspace=None, stream=None):
    """decode_attn over tokens starts[b] <= n < lens[b] (starts int32 [B] or None for 0)."""
    B, Hq, D = cache.B, cache.Hq, cache.D
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    need = decode_workspace_bytes(cache, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().loopvq_decode_attn_range(cache.ref(), layer, t, _ptr(q), _ptr(starts), _ptr(lens), max_len, scale,
                                          _ptr(out), _ptr(lse), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


class Bf16Cache:
    """A bf16 KV cache: k, v bf16 [B][Hkv][Nmax][D], keys already rotated (see include/loopvq.h)."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor, Hq: int):
        assert k.shape == v.shape and k.dtype == torch.bfloat16 and v.dtype == torch.bfloat16
        assert k.is_contiguous() and v.is_contiguous()
        self.k, self.v = k, v
        self.B, self.Hkv, self.Nmax, self.D = k.shape
        self.Hq = Hq
        self.desc = Bf16CacheDesc(self.B, self.Hkv, Hq, self.D, self.Nmax, k.data_ptr(), v.data_ptr())

    def ref(self):
        self.desc.k, self.desc.v = self.k.data_ptr(), self.v.data_ptr()
        return C.byref(self.desc)


def bf16_decode_workspace_bytes(cache: Bf16Cache, max_len: int) -> int:
    return lib().loopvq_bf16_decode_workspace_bytes(cache.ref(), max_len)


def bf16_decode_attn(cache: Bf16Cache, q: torch.Tensor, lens: torch.Tensor, max_len: int, starts=None,
                     scale: float = 0.0, out=None, lse=None, workspace=None, stream=None):
    """q bf16 [B][Hq][D]; attends tokens starts[b] <= n < lens[b]; returns (out, lse) like decode_attn."""
    B, Hq, D = cache.B, cache.Hq, cache.D
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    need = bf16_decode_workspace_bytes(cache, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().loopvq_bf16_decode_attn(cache.ref(), _ptr(q), _ptr(starts), _ptr(lens), max_len, scale, _ptr(out),
                                         _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream)))
    return out, lse


def merge2(out_a, lse_a, out_b, lse_b, out=None, lse=None, stream=None):
    """Log-sum-exp merge of two attentions over disjoint token sets; out may alias out_a / out_b."""
    D = out_a.shape[-1]
    rows = out_a.numel() // D
    if out is None:
        out = torch.empty_like(out_a)
    if lse is None:
        lse = torch.empty_like(lse_a)
    _check(lib().loopvq_merge2(_ptr(out_a), _ptr(lse_a), _ptr(out_b), _ptr(lse_b), rows, D, _ptr(out), _ptr(lse),
                               _stream(stream)))
    return out, lse


class Tasq:
    """TaSQ buffers of a cache (see include/loopvq.h): w fp32 [L][T][Hkv][D], perm int16 [L][NB][Hkv][D/2],
    sigma fp16 [L][T][B][Nmax] (written by tasq_encode)."""

    def __init__(self, cache: Cache, w=None, perm=None, device="cuda"):
        L = lib()
        nw, npm, ns = (L.loopvq_tasq_w_elems(cache.ref()), L.loopvq_tasq_perm_elems(cache.ref()),
                       L.loopvq_tasq_sigma_elems(cache.ref()))
        if nw == 0:
            raise LoopVQError(LOOPVQ_ERR_UNSUPPORTED, "this cache cannot be used with TaSQ (ncb = 1, c in {4, 8})")
        self.w = torch.ones(nw, dtype=torch.float32, device=device) if w is None else w.reshape(-1)
        self.perm = (torch.arange(cache.D // 2, dtype=torch.int16, device=device).repeat(npm // (cache.D // 2))
                     if perm is None else perm.reshape(-1))
        self.sigma = torch.ones(ns, dtype=torch.float16, device=device)
        self.desc = TasqDesc()

    def ref(self):
        self.desc.w, self.desc.perm, self.desc.sigma = self.w.data_ptr(), self.perm.data_ptr(), self.sigma.data_ptr()
        return C.byref(self.desc)


def tasq_encode(cache: Cache, tasq: Tasq, layer: int, block: int, xk, xv, b0: int = 0, tok0: int = 0, stream=None):
    """encode() with TaSQ; xk, xv as for encode()."""
    assert xk.shape == xv.shape and xk.stride() == xv.stride() and xk.dtype == xv.dtype
    Tc, nb, ntok, Hkv, D = xk.shape
    assert xk.stride(4) == 1
    dt = {torch.bfloat16: LOOPVQ_BF16, torch.float32: LOOPVQ_FP32}[xk.dtype]
    strides = (C.c_int64 * 4)(*xk.stride()[:4])
    _check(lib().loopvq_tasq_encode(cache.ref(), tasq.ref(), layer, block, _ptr(xk), _ptr(xv), dt, strides, b0, nb,
                                    tok0, ntok, _stream(stream)))


def tasq_decode_attn(cache: Cache, tasq: Tasq, layer: int, t: int, q, lens, max_len: int, scale: float = 0.0,
                     out=None, lse=None, workspace=None, stream=None):
    B, Hq, D = cache.B, cache.Hq, cache.D
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    need = decode_workspace_bytes(cache, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().loopvq_tasq_decode_attn(cache.ref(), tasq.ref(), layer, t, _ptr(q), _ptr(lens), max_len, scale,
                                         _ptr(out), _ptr(lse), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


class Window:
    """bf16 window of a coded cache (see include/loopvq.h): k_rot, k_pre, v bf16 [L][T][B][Hkv][W][D],
    fill and coded_end int32 [B] (coded_end starts at n_sink, fill at 0)."""

    def __init__(self, cache: Cache, n_sink: int = 8, n_recent: int = 64, device="cuda"):
        self.L, self.T, self.B, self.Hkv, self.Hq, self.D = cache.L, cache.T, cache.B, cache.Hkv, cache.Hq, cache.D
        self.n_sink, self.n_recent = n_sink, n_recent
        self.W = n_sink + n_recent + 8
        shape = (self.L, self.T, self.B, self.Hkv, self.W, self.D)
        self.k_rot = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.k_pre = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.v = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.fill = torch.zeros(self.B, dtype=torch.int32, device=device)
        self.coded_end = torch.full((self.B,), n_sink, dtype=torch.int32, device=device)
        self.desc = WindowDesc(self.L, self.T, self.B, self.Hkv, self.Hq, self.D, n_sink, n_recent)

    def ref(self):
        d = self.desc
        d.k_rot, d.k_pre, d.v = self.k_rot.data_ptr(), self.k_pre.data_ptr(), self.v.data_ptr()
        d.fill, d.coded_end = self.fill.data_ptr(), self.coded_end.data_ptr()
        return C.byref(d)


def window_advance(win: Window, cache: Cache, stream=None):
    _check(lib().loopvq_window_advance(win.ref(), cache.ref(), _stream(stream)))


def window_append(win: Window, layer: int, t: int, k_rot, k_pre, v, stream=None):
    """k_rot, k_pre, v: bf16 [B][Hkv][D] of the current token at (layer, loop step t)."""
    _check(lib().loopvq_window_append(win.ref(), layer, t, _ptr(k_rot), _ptr(k_pre), _ptr(v), _stream(stream)))


def window_workspace_bytes(win: Window, cache: Cache, max_coded: int) -> int:
    return lib().loopvq_window_workspace_bytes(win.ref(), cache.ref(), max_coded)


def window_decode_attn(win: Window, cache: Cache, layer: int, t: int, q, max_coded: int, scale: float = 0.0,
                       out=None, lse=None, workspace=None, stream=None):
    B, Hq, D = cache.B, cache.Hq, cache.D
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(window_workspace_bytes(win, cache, max_coded), 16), dtype=torch.uint8,
                                device=dev)
    _check(lib().loopvq_window_decode_attn(win.ref(), cache.ref(), layer, t, _ptr(q), max_coded, scale, _ptr(out),
                                           _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                           _stream(stream)))
    return out, lse


def window_append_decode_attn(win: Window, cache: Cache, layer: int, t: int, k_rot, k_pre, v, q, max_coded: int,
                              scale: float = 0.0, out=None, lse=None, workspace=None, stream=None):
    """window_append then window_decode_attn, in the decode call's launches (the merge kernel writes the
    token k_rot, k_pre, v, bf16 [B][Hkv][D], into slot fill - 1 and attends to it)."""
    B, Hq, D = cache.B, cache.Hq, cache.D
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(window_workspace_bytes(win, cache, max_coded), 16), dtype=torch.uint8,
                                device=dev)
    _check(lib().loopvq_window_append_decode_attn(win.ref(), cache.ref(), layer, t, _ptr(k_rot), _ptr(k_pre), _ptr(v),
                                                  _ptr(q), max_coded, scale, _ptr(out), _ptr(lse), _ptr(workspace),
                                                  workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


def dequant_debug(cache: Cache, layer: int, t: int, kv: int, b: int, tok0: int, ntok: int, apply_rope: bool = False,
                  out=None, stream=None):
    if out is None:
        out = torch.empty((cache.Hkv, ntok, cache.D), dtype=torch.float32, device="cuda")
    _check(lib().loopvq_dequant_debug(cache.ref(), layer, t, kv, b, tok0, ntok, int(bool(apply_rope)), _ptr(out),
                                      _stream(stream)))
    return out


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
