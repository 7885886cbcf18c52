"""The C-ABI library loads without a GPU, exports every declared symbol, and validates arguments
on the host before any launch."""
import ctypes as C
import os
import re

import pytest

import looped_lm_decode_b200 as LQ

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "loopvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(loopvq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 11
    lib = LQ.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(LQ.EXPORTS)
    assert lib.loopvq_abi_version() == 3


def _cache(**kw):
    args = dict(L=2, T=4, Tc=4, Hkv=16, Hq=16, D=128, c=4, K=256, B=8, Nmax=1024)
    args.update(kw)
    return LQ.Cache(**args, alloc=False)


def test_buffer_sizes():
    lib = LQ.lib()
    c = _cache()
    assert lib.loopvq_idx_words(c.ref()) == 2 * 1 * 8 * 16 * 1024 * 16
    assert lib.loopvq_codebook_elems(c.ref()) == 2 * 1 * 2 * 16 * 256 * 16
    assert lib.loopvq_slice_elems(c.ref()) == 2 * 4 * 2 * 16 * 256 * 4
    assert lib.loopvq_rope_elems(c.ref()) == 1024 * 128
    # 2*D/c bytes per token, head and block: 0.5 bit per element over Tc loop steps of K and V
    bits = lib.loopvq_idx_words(c.ref()) * 32 / (2 * 8 * 16 * 1024 * 4 * 2 * 128)
    assert bits == 0.5


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), 2), (dict(c=16), 2), (dict(c=64, Tc=1), 2), (dict(c=2), 2), (dict(Tc=3, T=6), 2), (dict(Hq=48), 2), (dict(Hq=17), 1),
    (dict(T=6), 1), (dict(K=300), 1), (dict(Nmax=1022), 1), (dict(B=0), 1)])
def test_shape_validation(kw, status):
    lib = LQ.lib()
    c = _cache(**kw)
    assert lib.loopvq_idx_words(c.ref()) == 0
    st = lib.loopvq_decode_attn(c.ref(), 0, 0, None, None, 0, 0.0, None, None, None, 0, None)
    assert st == status, lib.loopvq_last_error()


def test_argument_validation_before_launch():
    lib = LQ.lib()
    assert lib.loopvq_prepare(None, None) == 1
    assert b"NULL" in lib.loopvq_last_error()
    c = _cache()
    # fake, aligned, never-dereferenced pointers: every call must be refused on the host
    c.desc.idx = c.desc.slices = c.desc.rope = c.desc.codebook = 0x10000
    c.ref = lambda: C.byref(c.desc)          # keep the fake pointers in the descriptor
    fake = C.c_void_p(0x20000)
    assert lib.loopvq_decode_attn(c.ref(), 2, 0, fake, fake, 0, 0.0, fake, None, fake, 1 << 30, None) == 1
    assert b"layer" in lib.loopvq_last_error()
    assert lib.loopvq_decode_attn(c.ref(), 0, 4, fake, fake, 0, 0.0, fake, None, fake, 1 << 30, None) == 1
    assert lib.loopvq_decode_attn(c.ref(), 0, 0, fake, fake, 2000, 0.0, fake, None, fake, 1 << 30, None) == 1
    assert b"max_len" in lib.loopvq_last_error()
    need = lib.loopvq_decode_workspace_bytes(c.ref(), 1024)
    assert need > 0
    assert lib.loopvq_decode_attn(c.ref(), 0, 0, fake, fake, 1024, 0.0, fake, None, fake, need - 1, None) == 3
    assert lib.loopvq_decode_attn(c.ref(), 0, 0, fake, fake, 1024, 0.0, fake, None, None, need, None) == 3
    assert lib.loopvq_decode_attn(c.ref(), 0, 0, C.c_void_p(0x20002), fake, 1024, 0.0, fake, None, fake, need,
                                  None) == 1
    assert b"aligned" in lib.loopvq_last_error()
    assert lib.loopvq_dequant_debug(c.ref(), 0, 0, 2, 0, 0, 4, 0, fake, None) == 1
    assert lib.loopvq_dequant_debug(c.ref(), 0, 0, 0, 8, 0, 4, 0, fake, None) == 1
    strides = (C.c_int64 * 4)(1, 1, 1, 1)
    assert lib.loopvq_encode(c.ref(), 0, 1, fake, fake, 0, strides, 0, 1, 0, 4, None) == 1
    assert lib.loopvq_encode(c.ref(), 0, 0, fake, fake, 7, strides, 0, 1, 0, 4, None) == 1
    assert lib.loopvq_encode(c.ref(), 0, 0, fake, fake, 0, strides, 7, 2, 0, 4, None) == 1
    # an empty request is a no-op that succeeds without touching the device
    assert lib.loopvq_encode(c.ref(), 0, 0, None, None, 0, strides, 0, 0, 0, 0, None) == 0


def test_workspace_grows_with_context():
    lib = LQ.lib()
    c = _cache(Nmax=32768)
    a = lib.loopvq_decode_workspace_bytes(c.ref(), 1024)
    b = lib.loopvq_decode_workspace_bytes(c.ref(), 32768)
    assert 0 < a <= b
    assert lib.loopvq_decode_workspace_bytes(c.ref(), 40000) == 0


def _bf16_desc(**kw):
    args = dict(B=8, Hkv=16, Hq=16, D=128, Nmax=1024)
    args.update(kw)
    return LQ.Bf16CacheDesc(args["B"], args["Hkv"], args["Hq"], args["D"], args["Nmax"], 0x10000, 0x30000)


@pytest.mark.parametrize("kw,status", [(dict(D=96), 2), (dict(Hq=48), 2), (dict(Hq=17), 1), (dict(B=0), 1),
                                       (dict(Nmax=0), 1)])
def test_bf16_shape_validation(kw, status):
    lib = LQ.lib()
    d = _bf16_desc(**kw)
    fake = C.c_void_p(0x20000)
    assert lib.loopvq_bf16_decode_workspace_bytes(C.byref(d), 0) == 0
    st = lib.loopvq_bf16_decode_attn(C.byref(d), fake, None, fake, 0, 0.0, fake, None, fake, 1 << 30, None)
    assert st == status, lib.loopvq_last_error()


def test_bf16_argument_validation_before_launch():
    lib = LQ.lib()
    d = _bf16_desc()
    fake = C.c_void_p(0x20000)
    need = lib.loopvq_bf16_decode_workspace_bytes(C.byref(d), 1024)
    assert need > 0
    assert lib.loopvq_bf16_decode_attn(C.byref(d), fake, None, fake, 1025, 0.0, fake, None, fake, need, None) == 1
    assert b"max_len" in lib.loopvq_last_error()
    assert lib.loopvq_bf16_decode_attn(C.byref(d), fake, None, fake, 1024, 0.0, fake, None, fake, need - 1, None) == 3
    assert lib.loopvq_bf16_decode_attn(C.byref(d), fake, C.c_void_p(0x20002), fake, 1024, 0.0, fake, None, fake,
                                       need, None) == 1
    assert b"starts" in lib.loopvq_last_error()
    d.k = 0x10008
    assert lib.loopvq_bf16_decode_attn(C.byref(d), fake, None, fake, 1024, 0.0, fake, None, fake, need, None) == 1
    assert b"aligned" in lib.loopvq_last_error()
    d.k = None
    assert lib.loopvq_bf16_decode_attn(C.byref(d), fake, None, fake, 1024, 0.0, fake, None, fake, need, None) == 1
    assert b"NULL" in lib.loopvq_last_error()


def test_range_and_merge_validation_before_launch():
    lib = LQ.lib()
    c = _cache()
    c.desc.idx = c.desc.slices = c.desc.rope = c.desc.codebook = 0x10000
    c.ref = lambda: C.byref(c.desc)
    fake = C.c_void_p(0x20000)
    need = lib.loopvq_decode_workspace_bytes(c.ref(), 1024)
    assert lib.loopvq_decode_attn_range(c.ref(), 0, 0, fake, C.c_void_p(0x20001), fake, 1024, 0.0, fake, None, fake,
                                        need, None) == 1
    assert b"starts" in lib.loopvq_last_error()
    assert lib.loopvq_decode_attn_range(c.ref(), 0, 0, fake, fake, fake, 1024, 0.0, fake, None, fake, need - 1,
                                        None) == 3
    assert lib.loopvq_merge2(fake, fake, fake, fake, 4, 96, fake, fake, None) == 2
    assert lib.loopvq_merge2(fake, fake, fake, fake, -1, 128, fake, fake, None) == 1
    assert lib.loopvq_merge2(fake, None, fake, fake, 4, 128, fake, fake, None) == 1
    assert lib.loopvq_merge2(fake, fake, fake, fake, 4, 128, C.c_void_p(0x20002), fake, None) == 1
    assert lib.loopvq_merge2(None, None, None, None, 0, 128, None, None, None) == 0


def test_window_validation_before_launch():
    lib = LQ.lib()
    c = _cache()
    c.desc.idx = c.desc.slices = c.desc.rope = c.desc.codebook = 0x10000
    c.ref = lambda: C.byref(c.desc)
    fake = C.c_void_p(0x20000)
    w = LQ.WindowDesc(c.L, c.T, c.B, c.Hkv, c.Hq, c.D, 8, 64, 0x40000, 0x50000, 0x60000, 0x70000, 0x70100)
    assert lib.loopvq_window_slots(C.byref(w)) == 80
    need = lib.loopvq_window_workspace_bytes(C.byref(w), c.ref(), 1024)
    assert need > 0
    assert lib.loopvq_window_decode_attn(C.byref(w), c.ref(), 0, 0, fake, 1024, 0.0, fake, None, fake, need - 1,
                                         None) == 3
    assert lib.loopvq_window_decode_attn(C.byref(w), c.ref(), 0, 0, fake, 1025, 0.0, fake, None, fake, need,
                                         None) == 1
    assert lib.loopvq_window_append(C.byref(w), 2, 0, fake, fake, fake, None) == 1
    assert lib.loopvq_window_append(C.byref(w), 0, 0, fake, C.c_void_p(0x20008), fake, None) == 1
    # the fused call: a missing or misaligned token, a short workspace, a bad layer, all before any launch
    fused = lib.loopvq_window_append_decode_attn
    assert fused(C.byref(w), c.ref(), 0, 0, fake, None, fake, fake, 1024, 0.0, fake, None, fake, need, None) == 1
    assert b"required" in lib.loopvq_last_error()
    assert fused(C.byref(w), c.ref(), 0, 0, fake, C.c_void_p(0x20008), fake, fake, 1024, 0.0, fake, None, fake, need,
                 None) == 1
    assert fused(C.byref(w), c.ref(), 0, 0, fake, fake, fake, fake, 1024, 0.0, fake, None, fake, need - 1, None) == 3
    assert fused(C.byref(w), c.ref(), c.L, 0, fake, fake, fake, fake, 1024, 0.0, fake, None, fake, need, None) == 1
    w.n_recent = 60                                          # not a multiple of 8
    assert lib.loopvq_window_slots(C.byref(w)) == 0
    assert lib.loopvq_window_advance(C.byref(w), c.ref(), None) == 1
    assert b"multiples of 8" in lib.loopvq_last_error()
    w.n_recent, w.Hq = 64, 8                                 # shape differs from the cache's
    assert lib.loopvq_window_advance(C.byref(w), c.ref(), None) == 1
    assert b"differs" in lib.loopvq_last_error()
    w.Hq, w.fill = c.Hq, None
    assert lib.loopvq_window_advance(C.byref(w), c.ref(), None) == 1
    assert lib.loopvq_window_workspace_bytes(C.byref(w), c.ref(), 1024) == 0
    # the page roll stages the recent slots of one (layer, loop step, sequence, head) in shared memory:
    # 1024 x 128 bf16 = 256 KiB is more than a CTA can have, so the advance is refused before any launch
    w.fill, w.n_recent = 0x70000, 1024
    assert lib.loopvq_window_advance(C.byref(w), c.ref(), None) == 2
    assert b"shared memory" in lib.loopvq_last_error()
    w.n_recent = 904                                         # 904 x 128 x 2 = 231424 bytes: fits
    assert lib.loopvq_window_slots(C.byref(w)) == 8 + 904 + 8


def test_wait_limit_is_process_wide_and_settable():
    lib = LQ.lib()
    old = LQ.wait_limit_ns()
    assert old == 2_000_000_000
    LQ.set_wait_limit_ns(0)
    assert LQ.wait_limit_ns() == 0
    LQ.set_wait_limit_ns(old)
    assert lib.loopvq_wait_limit_ns() == old


def test_per_group_codebook_sizes_and_validation():
    """ncb = D/c multiplies the codebook and slice buffers; other values are refused."""
    lib = LQ.lib()
    c1 = _cache()
    cg = _cache()
    cg.desc.ncb = 128 // 4
    assert lib.loopvq_codebook_elems(cg.ref()) == 32 * lib.loopvq_codebook_elems(c1.ref())
    assert lib.loopvq_slice_elems(cg.ref()) == 32 * lib.loopvq_slice_elems(c1.ref())
    assert lib.loopvq_idx_words(cg.ref()) == lib.loopvq_idx_words(c1.ref())
    cg.desc.ncb = 7
    assert lib.loopvq_codebook_elems(cg.ref()) == 0
    assert lib.loopvq_prepare(cg.ref(), None) == 1
    assert b"ncb" in lib.loopvq_last_error()


def test_tasq_sizes_and_validation_before_launch():
    lib = LQ.lib()
    c = _cache()
    c.desc.idx = c.desc.slices = c.desc.rope = c.desc.codebook = 0x10000
    c.ref = lambda: C.byref(c.desc)
    assert lib.loopvq_tasq_w_elems(c.ref()) == 2 * 4 * 16 * 128
    assert lib.loopvq_tasq_perm_elems(c.ref()) == 2 * 1 * 16 * 64
    assert lib.loopvq_tasq_sigma_elems(c.ref()) == 2 * 4 * 8 * 1024
    fake = C.c_void_p(0x20000)
    t = LQ.TasqDesc(0x30000, 0x40000, 0x50000)
    need = lib.loopvq_decode_workspace_bytes(c.ref(), 1024)
    assert lib.loopvq_tasq_decode_attn(c.ref(), C.byref(t), 0, 4, fake, fake, 1024, 0.0, fake, None, fake, need,
                                       None) == 1
    assert lib.loopvq_tasq_decode_attn(c.ref(), None, 0, 0, fake, fake, 1024, 0.0, fake, None, fake, need, None) == 1
    t.perm = 0x40001                                                       # misaligned int16 array
    assert lib.loopvq_tasq_decode_attn(c.ref(), C.byref(t), 0, 0, fake, fake, 1024, 0.0, fake, None, fake, need,
                                       None) == 1
    assert b"misaligned" in lib.loopvq_last_error()
    t.perm = 0x40000
    strides = (C.c_int64 * 4)(1, 1, 1, 1)
    assert lib.loopvq_tasq_encode(c.ref(), C.byref(t), 0, 1, fake, fake, 0, strides, 0, 1, 0, 4, None) == 1
    assert b"block" in lib.loopvq_last_error()
    c16 = _cache(c=16, Tc=1)
    assert lib.loopvq_tasq_w_elems(c16.ref()) == 0
    c16.desc.idx = c16.desc.slices = c16.desc.rope = c16.desc.codebook = 0x10000
    c16.ref = lambda: C.byref(c16.desc)
    assert lib.loopvq_tasq_decode_attn(c16.ref(), C.byref(t), 0, 0, fake, fake, 1024, 0.0, fake, None, fake, need,
                                       None) == 2
