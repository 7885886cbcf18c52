"""loopvq_decode_attn_noalloc: decode attention for callers that cannot allocate device memory.

Some callers have no way to hand the library a device workspace: plain C hosts
without a device allocator, plug-ins whose host application owns the whole
device through its own allocator, and serving loops that must not call
cudaMalloc because it can synchronise the device.  For them the library keeps
the split scratch in a fixed array compiled into it.  This test calls that entry
point through the C ABI twice in a row and checks it against the entry point that
takes a caller workspace, and checks that a call needing more scratch than the
array holds is refused before anything runs.

The file name sorts last so that a run stopping at the first failure has already
run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import looped_lm_decode_b200 as LQ
from synth import WORKLOADS, queries
from synth import gpu as SG
from tests.helpers import attn_tolerance_ok

pytestmark = pytest.mark.gpu


def _noalloc(cache, layer, t, q, lens, max_len):
    out = torch.empty((cache.B, cache.Hq, cache.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((cache.B, cache.Hq), dtype=torch.float32, device="cuda")
    st = LQ.lib().loopvq_decode_attn_noalloc(cache.ref(), layer, t, C.c_void_p(q.data_ptr()),
                                             C.c_void_p(lens.data_ptr()), max_len, 0.0, C.c_void_p(out.data_ptr()),
                                             C.c_void_p(lse.data_ptr()),
                                             C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, LQ.lib().loopvq_last_error()
    return out, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    w = WORKLOADS["ctx4k"].replace(L=2, B=3, Hkv=4, Hq=8, Nmax=2048)
    cache = LQ.Cache(w.L, w.T, w.Tc, w.Hkv, w.Hq, w.D, w.c, w.K, w.B, w.Nmax, w.theta)
    SG.fill_codebook(w, cache.codebook)
    LQ.prepare(cache)
    per = w.B * w.Hkv * w.Nmax * cache.NP
    for layer in range(w.L):
        SG.fill_idx(w, layer, 0, cache.idx[layer * per:(layer + 1) * per])
    lens = torch.tensor([2048, 1000, 37], dtype=torch.int32, device="cuda")
    assert LQ.decode_workspace_bytes(cache, 2048) <= LQ.lib().loopvq_noalloc_scratch_bytes()
    for layer, t in [(0, 1), (1, 3)]:
        q = torch.from_numpy(queries(w, layer, t).view(np.int16)).cuda()
        ref, lref = LQ.decode_attn(cache, layer, t, q, lens, 2048)
        got, lgot = _noalloc(cache, layer, t, q, lens, 2048)
        torch.cuda.synchronize()
        ok, msg = attn_tolerance_ok(got.cpu().numpy(), ref.cpu().numpy(), lgot.cpu().numpy(), lref.cpu().numpy())
        assert ok, f"(layer {layer}, t {t}): {msg}"


def test_noalloc_rejects_calls_larger_than_its_scratch():
    # the partial records scale with (sequences x KV heads + CTAs) x query heads per KV head
    c = LQ.Cache(1, 4, 4, 16, 32, 128, 4, 256, 1024, 32768, alloc=False)
    need = LQ.lib().loopvq_decode_workspace_bytes(c.ref(), 32768)
    assert need > LQ.lib().loopvq_noalloc_scratch_bytes()
    # aligned addresses that are never dereferenced: the call must be refused before any launch
    c.desc.idx = c.desc.slices = c.desc.rope = c.desc.codebook = 0x10000
    fake = C.c_void_p(0x20000)
    st = LQ.lib().loopvq_decode_attn_noalloc(C.byref(c.desc), 0, 0, fake, fake, 32768, 0.0, fake, None, None)
    assert st == 3
    assert b"scratch" in LQ.lib().loopvq_last_error()
