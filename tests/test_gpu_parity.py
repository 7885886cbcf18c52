"""GPU path vs the CPU checker, element by element, through the C ABI.

Bars: codes bit-exact (a mismatch is allowed only as a near-tie whose two fp64
distances differ by < 1e-5 relative, and is counted); reconstruction bit-exact;
attention max|out - ref| <= 2e-3 * ||ref||_inf per call tensor and
|lse - lse_ref| <= 1e-3.  Inputs are seeded synthetic data from synth/; the
checker never sees anything the GPU produced except the outputs it is compared with.
"""
import math

import numpy as np
import pytest
import torch

import looped_lm_decode_b200 as LQ
from oracle import oracle as O
from synth import (WORKLOADS, kv_loops, codebook, codebooks, queries, lengths, random_indices, bf16_bits_to_f32)
from synth import gpu as SG
from tests.helpers import (pack_words, unpack_words, words_view, codebook_view, make_cache, np_codebook_f32,
                           attn_tolerance_ok)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": WORKLOADS["tiny"],
    "ctx": WORKLOADS["ctx4k"].replace(L=2, B=3, Hkv=2, Hq=2, Nmax=1024),
    "gqa": WORKLOADS["gqa16k"].replace(L=1, B=2, Hkv=2, Hq=8, Nmax=512),
    "deep": WORKLOADS["deep32"].replace(L=1, T=8, B=2, Hkv=3, Hq=3, Nmax=256),
    "d64c8": WORKLOADS["tiny"].replace(c=8, Hq=2, B=2, Nmax=128),
    "qpk2": WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=2, Hq=4, Nmax=256),
    # plain per-loop-step coding (CQ): Tc = 1, c = G, on the same kernels
    "cq16": WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=2, Hq=2, Nmax=256, c=16, Tc=1),
    "cq32g": WORKLOADS["gqa16k"].replace(L=1, B=2, Hkv=1, Hq=4, Nmax=128, c=32, Tc=1),
    "cq16d64": WORKLOADS["tiny"].replace(c=16, Tc=2, B=2, Hq=2, Hkv=2, Nmax=128),
    # one codebook per channel group (ncb = D/c)
    "pg4": WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=2, Hq=2, Nmax=256, ncb=32),
    "pg8gqa": WORKLOADS["gqa16k"].replace(L=1, B=2, Hkv=1, Hq=4, Nmax=128, ncb=16),
    "pgd64": WORKLOADS["tiny"].replace(B=2, Hq=2, Hkv=2, Nmax=128, ncb=16),
    "pgcq16": WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=2, Hq=2, Nmax=128, c=16, Tc=1, ncb=8),
}


def _dec(q, ik, iv, Ek, Ev, *args):
    """The checker's decode with a shared ([K][G]) or per-group ([NCB][K][G]) codebook."""
    return (O.decode_pg if np.ndim(Ek) == 3 else O.decode)(q, ik, iv, Ek, Ev, *args)


def _enc(x, E, c):
    return (O.encode_pg if np.ndim(E) == 3 else O.encode)(x, E, c)


def _deq(idx, E, c, Tc, m):
    return (O.dequant_pg if np.ndim(E) == 3 else O.dequant)(idx, E, c, Tc, m)


def _dist(x, E, c, n, g, r):
    return (O.dist64_pg if np.ndim(E) == 3 else O.dist64)(x, E, c, n, g, r)


def _upload_random_codes(w, cache):
    codes = {}
    for layer in range(w.L):
        for blk in range(w.NB):
            for b in range(w.B):
                for h in range(w.Hkv):
                    ik = random_indices(w, layer, blk, 0, b, h, range(w.Nmax))
                    iv = random_indices(w, layer, blk, 1, b, h, range(w.Nmax))
                    codes[(layer, blk, b, h)] = (ik, iv)
                    words = pack_words(ik, iv, cache.NP).view(np.int32)
                    words_view(cache, layer, blk, b, h).copy_(torch.from_numpy(words))
    return codes


def _oracle_call(w, codes, layer, t, q_bits, lens, scale):
    blk, m = t // w.Tc, t % w.Tc
    qpk = w.Hq // w.Hkv
    outs = np.zeros((w.B, w.Hq, w.D))
    lses = np.zeros((w.B, w.Hq))
    for b in range(w.B):
        for hq in range(w.Hq):
            h = hq // qpk
            ik, iv = codes[(layer, blk, b, h)]
            n = int(lens[b])
            o, l = _dec(bf16_bits_to_f32(q_bits[b, hq]).astype(np.float64), ik[:n], iv[:n],
                            np_codebook_f32(w, layer, blk, 0, h), np_codebook_f32(w, layer, blk, 1, h),
                            w.c, w.Tc, m, w.theta, scale)
            outs[b, hq], lses[b, hq] = o, l
    return outs, lses


def _gpu_call(cache, layer, t, q_bits, lens, max_len, scale=0.0):
    q = torch.from_numpy(q_bits.view(np.int16)).cuda()
    lt = torch.from_numpy(np.asarray(lens, np.int32)).cuda()
    out, lse = LQ.decode_attn(cache, layer, t, q, lt, max_len, scale)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def _lens(w, kind):
    if kind == "full":
        return np.full(w.B, w.Nmax, np.int32)
    rng = np.random.default_rng(7)
    return rng.integers(1, w.Nmax + 1, w.B).astype(np.int32)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("lens_kind", ["full", "ragged"])
def test_decode_parity_small(name, lens_kind):
    w = SMALL[name]
    cache = make_cache(w)
    codes = _upload_random_codes(w, cache)
    lens = _lens(w, lens_kind)
    scale = 1.0 / math.sqrt(w.D)
    for layer in range(w.L):
        for t in range(w.T):
            qb = queries(w, layer, t)
            out, lse = _gpu_call(cache, layer, t, qb, lens, int(lens.max()))
            ref, lref = _oracle_call(w, codes, layer, t, qb, lens, scale)
            ok, msg = attn_tolerance_ok(out, ref, lse, lref)
            assert ok, f"{name} layer {layer} t {t}: {msg}"


@pytest.mark.parametrize("name", ["ctx", "gqa", "cq16"])
@pytest.mark.parametrize("gain", [8.0, 0.0])
def test_decode_peaky_and_flat_queries(name, gain):
    """q x 8 makes the softmax peaky (large max-rescale traffic); q = 0 gives the mean of values.  "ctx"
    runs the one-head-per-KV-head kernel, "cq16" the same kernel with groups of 16 channels, "gqa" the
    4-heads-per-KV-head kernel."""
    w = SMALL[name]
    cache = make_cache(w)
    codes = _upload_random_codes(w, cache)
    lens = _lens(w, "ragged")
    layer = min(1, w.L - 1)
    qb = queries(w, layer, 2, gain=gain)
    out, lse = _gpu_call(cache, layer, 2, qb, lens, int(lens.max()))
    ref, lref = _oracle_call(w, codes, layer, 2, qb, lens, 1 / math.sqrt(w.D))
    ok, msg = attn_tolerance_ok(out, ref, lse, lref)
    assert ok, msg


@pytest.mark.parametrize("name", ["ctx", "gqa", "cq16"])
def test_decode_edge_lengths(name):
    w = SMALL[name].replace(B=8)
    N = w.Nmax
    cache = make_cache(w)
    codes = _upload_random_codes(w, cache)
    lens = np.array([0, 1, 3, 4, 5, N // 2 - 1, N - 1, N], np.int32)
    qb = queries(w, 0, 3)
    out, lse = _gpu_call(cache, 0, 3, qb, lens, N)
    ref, lref = _oracle_call(w, codes, 0, 3, qb, lens, 1 / math.sqrt(w.D))
    ok, msg = attn_tolerance_ok(out, ref, lse, lref)
    assert ok, msg
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()
    # lengths above max_len are clamped to it
    cut = N * 3 // 5
    out2, lse2 = _gpu_call(cache, 0, 3, qb, np.full(8, N, np.int32), cut)
    ref2, lref2 = _oracle_call(w, codes, 0, 3, qb, np.full(8, cut, np.int32), 1 / math.sqrt(w.D))
    ok, msg = attn_tolerance_ok(out2, ref2, lse2, lref2)
    assert ok, msg
    # max_len = 0: nothing to attend
    out3, lse3 = _gpu_call(cache, 0, 3, qb, lens, 0)
    assert (out3 == 0).all() and np.isneginf(lse3).all()


@pytest.mark.parametrize("w", [WORKLOADS["ctx4k"].replace(L=1, B=3, Hkv=2, Hq=2, Nmax=20),
                               WORKLOADS["ctx4k"].replace(L=1, B=3, Hkv=2, Hq=2, Nmax=20, c=16, Tc=1),
                               WORKLOADS["gqa16k"].replace(L=1, B=3, Hkv=1, Hq=4, Nmax=12),
                               WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=1, Hq=1, Nmax=4)],
                         ids=["mha-nmax20", "mha-c16-nmax20", "gqa-nmax12", "mha-nmax4"])
def test_decode_short_caches(w):
    """Caches shorter than a 16-token tile (and one below the 8 positions the one- and four-head kernels
    need, which takes the general kernel): partial tiles, zero-filled index copies, RoPE rows near Nmax."""
    cache = make_cache(w)
    codes = _upload_random_codes(w, cache)
    lens = np.array([w.Nmax, 7, 3][:w.B], np.int32)
    for t in (0, 3):
        qb = queries(w, 0, t)
        out, lse = _gpu_call(cache, 0, t, qb, lens, w.Nmax)
        ref, lref = _oracle_call(w, codes, 0, t, qb, lens, 1 / math.sqrt(w.D))
        ok, msg = attn_tolerance_ok(out, ref, lse, lref)
        assert ok, f"t {t}: {msg}"


@pytest.mark.parametrize("name", ["tiny", "ctx", "gqa"])
def test_decode_explicit_scale(name):
    w = SMALL[name]
    cache = make_cache(w)
    codes = _upload_random_codes(w, cache)
    lens = np.array([200, w.Nmax, 77][:w.B], np.int32)
    qb = queries(w, 0, 1)
    out, lse = _gpu_call(cache, 0, 1, qb, lens, w.Nmax, scale=0.3)
    ref, lref = _oracle_call(w, codes, 0, 1, qb, lens, 0.3)
    ok, msg = attn_tolerance_ok(out, ref, lse, lref)
    assert ok, msg


@pytest.mark.parametrize("name", ["tiny", "deep", "gqa", "pg4", "pgd64", "pgcq16"])
def test_dequant_debug_bit_exact(name):
    w = SMALL[name]
    cache = make_cache(w)
    codes = _upload_random_codes(w, cache)
    b = w.B - 1
    for t in range(w.T):
        blk, m = t // w.Tc, t % w.Tc
        for kv in range(2):
            rec = LQ.dequant_debug(cache, 0, t, kv, b, 4, 60, apply_rope=False).cpu().numpy()
            for h in range(w.Hkv):
                ref = _deq(codes[(0, blk, b, h)][kv][4:64], np_codebook_f32(w, 0, blk, kv, h), w.c, w.Tc, m)
                np.testing.assert_array_equal(rec[h].astype(np.float64), ref)
        rot = LQ.dequant_debug(cache, 0, t, 0, b, 100, 28, apply_rope=True).cpu().numpy()
        for h in range(w.Hkv):
            k = _deq(codes[(0, blk, b, h)][0][100:128], np_codebook_f32(w, 0, blk, 0, h), w.c, w.Tc, m)
            ref = O.rope(k, w.theta, 100)
            np.testing.assert_allclose(rot[h], ref, rtol=0, atol=2e-5 * np.abs(ref).max())


def _x_block(w, layer, blk, kv, dtype):
    x = kv_loops(w, layer, kv, blk * w.Tc, blk * w.Tc + w.Tc - 1, range(w.B), range(w.Nmax), range(w.Hkv),
                 dtype="bf16" if dtype == "bf16" else "f32")
    return x          # [Tc][B][N][Hkv][D]


def _to_dev(x, dtype):
    if dtype == "bf16":
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def _check_codes(w, x_np, dtype, E, codes_gpu, b, h, kv):
    xf = bf16_bits_to_f32(x_np) if dtype == "bf16" else x_np
    xb = np.ascontiguousarray(xf[:, b, :, h, :])
    ref = _enc(xb, E, w.c)
    mism = np.argwhere(codes_gpu != ref)
    ties = 0
    for n, g in mism:
        dg = _dist(xb, E, w.c, n, g, int(codes_gpu[n, g]))
        do = _dist(xb, E, w.c, n, g, int(ref[n, g]))
        assert abs(dg - do) <= 1e-5 * max(dg, do), (b, h, kv, n, g, dg, do)
        ties += 1
    return ties


@pytest.mark.parametrize("name,dtype", [("tiny", "bf16"), ("tiny", "f32"), ("ctx", "bf16"), ("gqa", "bf16"),
                                        ("deep", "bf16"), ("d64c8", "f32"), ("cq16", "bf16"), ("cq16", "f32"),
                                        ("cq32g", "bf16"), ("cq16d64", "bf16"), ("pg4", "bf16"), ("pg8gqa", "bf16"),
                                        ("pgd64", "f32"), ("pgcq16", "bf16")])
def test_encode_parity(name, dtype):
    w = SMALL[name]
    if name == "ctx":
        w = w.replace(Nmax=256)
    cache = make_cache(w)
    ties = 0
    for layer in range(w.L):
        for blk in range(w.NB):
            xk = _x_block(w, layer, blk, 0, dtype)
            xv = _x_block(w, layer, blk, 1, dtype)
            LQ.encode(cache, layer, blk, _to_dev(xk, dtype), _to_dev(xv, dtype))
            torch.cuda.synchronize()
            for b in range(w.B):
                for h in range(w.Hkv):
                    words = words_view(cache, layer, blk, b, h).cpu().numpy().view(np.uint32)
                    ck, cv = unpack_words(words, w.Nmax, cache.NP)
                    ties += _check_codes(w, xk, dtype, np_codebook_f32(w, layer, blk, 0, h), ck, b, h, 0)
                    ties += _check_codes(w, xv, dtype, np_codebook_f32(w, layer, blk, 1, h), cv, b, h, 1)
    print(f"near-ties: {ties}")


@pytest.mark.parametrize("name", ["ctx", "pg4"])
def test_encode_partial_ranges_and_strides(name):
    """Encoding sub-ranges (b0, tok0 offsets, ragged token counts, strided input) writes exactly those words.
    "pg4" has one codebook per channel group: the tensor-core encoder writes each group's bytes."""
    w = SMALL[name].replace(Nmax=128, L=1, B=3)
    cache = make_cache(w)
    sentinel = torch.full_like(cache.idx, -1)
    cache.idx.copy_(sentinel)
    xk = _x_block(w, 0, 0, 0, "bf16")
    xv = _x_block(w, 0, 0, 1, "bf16")
    dk, dv = _to_dev(xk, "bf16"), _to_dev(xv, "bf16")
    # sequences 1..2, tokens 37..37+50, from a strided view
    LQ.encode(cache, 0, 0, dk[:, 1:3, 37:87], dv[:, 1:3, 37:87], b0=1, tok0=37)
    torch.cuda.synchronize()
    for b in range(w.B):
        for h in range(w.Hkv):
            words = words_view(cache, 0, 0, b, h).cpu().numpy().view(np.uint32)
            ck, cv = unpack_words(words, w.Nmax, cache.NP)
            wr = np.ones(w.Nmax, bool) if b in (1, 2) else np.zeros(w.Nmax, bool)
            wr[:37] = False
            wr[87:] = False
            untouched = words.reshape(w.Nmax // 4, cache.NP, 4).transpose(0, 2, 1).reshape(w.Nmax, cache.NP)
            assert (untouched[~wr] == 0xFFFFFFFF).all()
            if wr.any():
                ref_k = _enc(np.ascontiguousarray(bf16_bits_to_f32(xk)[:, b, 37:87, h, :]),
                             np_codebook_f32(w, 0, 0, 0, h), w.c)
                ref_v = _enc(np.ascontiguousarray(bf16_bits_to_f32(xv)[:, b, 37:87, h, :]),
                             np_codebook_f32(w, 0, 0, 1, h), w.c)
                np.testing.assert_array_equal(ck[37:87], ref_k)
                np.testing.assert_array_equal(cv[37:87], ref_v)


def test_generator_twins_agree():
    """The CUDA generator reproduces the numpy generator bit for bit (spot checks)."""
    w = WORKLOADS["ctx32k"].replace(L=1, B=2, Nmax=64)
    out = torch.empty((2, w.B, w.Nmax, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
    SG.fill_kv(w, 0, 1, 2, 3, out)
    ref = kv_loops(w, 0, 1, 2, 3, range(w.B), range(w.Nmax), range(w.Hkv))
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), ref)
    q = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    SG.fill_q(w, 0, 3, q)
    np.testing.assert_array_equal(q.view(torch.int16).cpu().numpy().view(np.uint16), queries(w, 0, 3))
    w4 = WORKLOADS["deep32"].replace(L=2, Hkv=3, Hq=3, Nmax=64)
    cache = LQ.Cache(w4.L, w4.T, w4.Tc, w4.Hkv, w4.Hq, w4.D, w4.c, w4.K, w4.B, w4.Nmax, w4.theta)
    SG.fill_codebook(w4, cache.codebook)
    for (layer, blk, kv, h) in [(0, 0, 0, 0), (1, 7, 1, 2), (1, 3, 0, 1)]:
        got = codebook_view(cache, layer, blk, kv, h).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, codebook(w4, layer, blk, kv, h).reshape(-1))
    SG.fill_idx(w4, 1, 5, cache.idx[: w4.B * w4.Hkv * w4.Nmax * cache.NP])
    words = cache.idx[: w4.B * w4.Hkv * w4.Nmax * cache.NP].cpu().numpy().view(np.uint32)
    per = w4.Nmax * cache.NP
    for b, h in [(0, 0), (1, 2)]:
        run = words[(b * w4.Hkv + h) * per:(b * w4.Hkv + h + 1) * per]
        ck, cv = unpack_words(run, w4.Nmax, cache.NP)
        np.testing.assert_array_equal(ck, random_indices(w4, 1, 5, 0, b, h, range(w4.Nmax)))
        np.testing.assert_array_equal(cv, random_indices(w4, 1, 5, 1, b, h, range(w4.Nmax)))


def test_generator_twins_agree_per_group_codebooks():
    """The CUDA generator's per-group codebooks equal the numpy ones bit for bit."""
    w = WORKLOADS["ctx4k"].replace(L=2, Hkv=2, Hq=2, B=1, Nmax=64, ncb=32)
    cache = LQ.Cache(w.L, w.T, w.Tc, w.Hkv, w.Hq, w.D, w.c, w.K, w.B, w.Nmax, w.theta, ncb=w.ncb)
    SG.fill_codebook(w, cache.codebook)
    for (layer, blk, kv, h) in [(0, 0, 0, 0), (1, 0, 1, 1)]:
        got = codebook_view(cache, layer, blk, kv, h).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, codebooks(w, layer, blk, kv, h).reshape(-1))
