"""Faults a kernel finds on the device reach the caller through loopvq_fault_check.

Neither test faults, traps or hangs the GPU.  The encoder's bounded wait is made to run out by a zero
limit (it gives up at its first unsuccessful poll, then waits, bounded, for the contraction it already
issued before releasing its tensor memory); the window roll is given a sequence whose coded cache is
full.  Each test then checks the status, that the fault word was cleared, and that the library still
computes correct results on the same context.
"""
import numpy as np
import pytest
import torch

import looped_lm_decode_b200 as LQ
from looped_lm_decode_b200.loopvq import LOOPVQ_ERR_OVERFLOW, LOOPVQ_ERR_TIMEOUT
from oracle import oracle as O
from synth import WORKLOADS, kv_loops, bf16_bits_to_f32
from synth import gpu as SG
from tests.helpers import make_cache, np_codebook_f32, unpack_words, words_view

pytestmark = pytest.mark.gpu


def _codes_match(w, cache, layer, blk, b, h, tok):
    """GPU codes of tokens `tok` equal the checker's encode (near-ties under the 1e-5 rule allowed)."""
    words = words_view(cache, layer, blk, b, h).cpu().numpy().view(np.uint32)
    ck, cv = unpack_words(words, w.Nmax, cache.NP)
    for kv, codes in ((0, ck), (1, cv)):
        x = kv_loops(w, layer, kv, blk * w.Tc, blk * w.Tc + w.Tc - 1, [b], tok, [h])[:, 0, :, 0, :]
        xf = np.ascontiguousarray(bf16_bits_to_f32(x))
        E = np_codebook_f32(w, layer, blk, kv, h)
        ref = O.encode(xf, E, w.c)
        for i, g in zip(*np.nonzero(codes[tok] != ref)):
            dg = O.dist64(xf, E, w.c, int(i), int(g), int(codes[tok][i, g]))
            do = O.dist64(xf, E, w.c, int(i), int(g), int(ref[i, g]))
            assert abs(dg - do) <= 1e-5 * max(dg, do), (kv, i, g)


def test_encode_wait_that_runs_out_is_reported():
    w = WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=4, Hq=4, Nmax=1024)
    cache = make_cache(w)
    LQ.fault_check()                                   # nothing pending from earlier calls
    xs = []
    for kv in range(2):
        x = torch.empty((w.Tc, w.B, w.Nmax, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
        SG.fill_kv(w, 0, kv, 0, w.Tc - 1, x)
        xs.append(x)
    old = LQ.wait_limit_ns()
    LQ.set_wait_limit_ns(0)
    try:
        LQ.encode(cache, 0, 0, xs[0], xs[1])           # tensor-core path (bf16 input)
        with pytest.raises(LQ.LoopVQError) as err:
            LQ.fault_check()
        assert err.value.status == LOOPVQ_ERR_TIMEOUT
    finally:
        LQ.set_wait_limit_ns(old)
    LQ.fault_check()                                   # the check cleared the word
    # same context, default bound: the encoder runs to completion and its codes are the checker's
    LQ.encode(cache, 0, 0, xs[0], xs[1])
    LQ.fault_check()
    tok = np.array([0, 1, 2, 127, 128, 500, 1023])
    for b, h in ((0, 0), (1, 3)):
        _codes_match(w, cache, 0, 0, b, h, tok)


def test_window_roll_without_room_is_reported():
    """Sequence 0's coded cache is full (coded_end + 8 > Nmax), sequence 1's has room: one advance rolls
    sequence 1 only, sets the overflow fault, and leaves sequence 0's counters, slots and codes alone."""
    w = WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=2, Hq=2, Nmax=44)
    cache = make_cache(w)
    win = LQ.Window(cache, n_sink=8, n_recent=16)      # W = 32 slots
    gen = torch.Generator(device="cuda").manual_seed(7)
    for buf in (win.k_rot, win.k_pre, win.v):
        buf.copy_(torch.randn(buf.shape, generator=gen, device="cuda").to(torch.bfloat16))
    win.fill.fill_(win.W)
    win.coded_end.copy_(torch.tensor([40, 32], dtype=torch.int32))
    LQ.fault_check()
    before = {k: getattr(win, k).clone() for k in ("k_rot", "k_pre", "v")}
    idx_before = cache.idx.clone()
    LQ.window_advance(win, cache)
    with pytest.raises(LQ.LoopVQError) as err:
        LQ.fault_check()
    assert err.value.status == LOOPVQ_ERR_OVERFLOW
    LQ.fault_check()
    assert win.coded_end.tolist() == [40, 40]
    assert win.fill.tolist() == [win.W, win.W - 8 + 1]
    for k, old in before.items():
        new = getattr(win, k)
        assert torch.equal(new[:, :, 0], old[:, :, 0]), k                      # sequence 0 untouched
        assert torch.equal(new[:, :, 1, :, 8:8 + 16], old[:, :, 1, :, 16:32]), k  # sequence 1 shifted
    # sequence 0's codes are unchanged; sequence 1's page (its slots 8..15) became tokens 32..39
    for h in range(w.Hkv):
        assert torch.equal(words_view(cache, 0, 0, 0, h), words_view(_as_cache(cache, idx_before), 0, 0, 0, h))
        words = words_view(cache, 0, 0, 1, h).cpu().numpy().view(np.uint32)
        ck, cv = unpack_words(words, w.Nmax, cache.NP)
        for kv, codes, src in ((0, ck, before["k_pre"]), (1, cv, before["v"])):
            x = src[0, 0:w.Tc, 1, h, 8:16].view(torch.int16).cpu().numpy().view(np.uint16)
            ref = O.encode(bf16_bits_to_f32(x), np_codebook_f32(w, 0, 0, kv, h), w.c)
            np.testing.assert_array_equal(codes[32:40], ref)


class _as_cache:
    """A cache view whose index buffer is a saved copy (for words_view)."""

    def __init__(self, cache, idx):
        self.Nmax, self.NP, self.NB, self.B, self.Hkv = cache.Nmax, cache.NP, cache.NB, cache.B, cache.Hkv
        self.idx = idx
