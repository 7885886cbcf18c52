"""bf16 decode kernel, coded token ranges and the bf16-window + coded-cache layout vs the CPU checker.

The pages keep the first n_s (sink) and last n_r (recent) tokens of a request in bf16, with keys
stored already rotated, and code the rest (LoopVQ paper, Sec. 4.3 "Cache layout"); one kernel attends
to each part and the results are combined through their log-sum-exps ("Attention").  The bars are
those of the coded decode: max|out - ref| <= 2e-3 * ||ref||_inf, |lse - lse_ref| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import looped_lm_decode_b200 as LQ
from oracle import oracle as O
from synth import WORKLOADS, kv_loops, queries, random_indices, bf16_bits_to_f32
from tests.helpers import pack_words, words_view, make_cache, np_codebook_f32, attn_tolerance_ok

pytestmark = pytest.mark.gpu

N_SINK, N_RECENT = 8, 64            # the pages' serving setting (Sec. 5.3)


def _bf16_cache_bits(w, layer, t, n):
    """bf16 bits [B][Hkv][n][D] of keys (kv = 0) and values (kv = 1): seeded data standing for a bf16
    cache whose keys were rotated when written."""
    out = []
    for kv in range(2):
        x = kv_loops(w, layer, kv, t, t, range(w.B), range(n), range(w.Hkv))[0]     # [B][n][Hkv][D]
        out.append(np.ascontiguousarray(x.transpose(0, 2, 1, 3)))
    return out


def _dev_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)


def _dev_i32(x):
    return torch.from_numpy(np.asarray(x, np.int32)).cuda()


BF16_SHAPES = {
    "mha128": WORKLOADS["ctx4k"].replace(B=3, Hkv=2, Hq=2, Nmax=700),
    "gqa4": WORKLOADS["gqa16k"].replace(B=2, Hkv=2, Hq=8, Nmax=512),
    "qpk8": WORKLOADS["ctx4k"].replace(B=2, Hkv=1, Hq=8, Nmax=300),
    "d64qpk2": WORKLOADS["tiny"].replace(B=3, Hkv=2, Hq=4, Nmax=260),
}


@pytest.mark.parametrize("name", list(BF16_SHAPES))
@pytest.mark.parametrize("gain", [1.0, 8.0])
def test_bf16_decode_parity(name, gain):
    w = BF16_SHAPES[name]
    kb, vb = _bf16_cache_bits(w, 0, 1, w.Nmax)
    cache = LQ.Bf16Cache(_dev_bits(kb), _dev_bits(vb), w.Hq)
    rng = np.random.default_rng(11)
    lens = rng.integers(0, w.Nmax + 1, w.B).astype(np.int32)
    lens[0] = w.Nmax
    if w.B > 2:
        lens[2] = 1
    starts = np.array([rng.integers(0, max(int(l), 1)) for l in lens], np.int32)
    starts[-1] = lens[-1]                                   # an empty range
    qb = queries(w, 0, 1, gain=gain)
    max_len = int(lens.max())
    for with_starts in (False, True):
        st = starts if with_starts else np.zeros(w.B, np.int32)
        out, lse = LQ.bf16_decode_attn(cache, _dev_bits(qb), _dev_i32(lens), max_len,
                                       starts=_dev_i32(st) if with_starts else None)
        torch.cuda.synchronize()
        out, lse = out.cpu().numpy(), lse.cpu().numpy()
        ref = np.zeros((w.B, w.Hq, w.D))
        lref = np.zeros((w.B, w.Hq))
        qpk = w.Hq // w.Hkv
        for b in range(w.B):
            for hq in range(w.Hq):
                h = hq // qpk
                a, e = int(st[b]), int(lens[b])
                ref[b, hq], lref[b, hq] = O.attention(bf16_bits_to_f32(qb[b, hq]).astype(np.float64),
                                                      bf16_bits_to_f32(kb[b, h, a:e]), bf16_bits_to_f32(vb[b, h, a:e]),
                                                      1 / math.sqrt(w.D))
        ok, msg = attn_tolerance_ok(out, ref, lse, lref)
        assert ok, f"{name} starts={with_starts}: {msg}"


CODED = WORKLOADS["ctx4k"].replace(L=1, B=4, Hkv=2, Hq=2, Nmax=512)
CODED_GQA = WORKLOADS["gqa16k"].replace(L=1, B=2, Hkv=2, Hq=8, Nmax=256)


def _coded_cache(w, layer=0):
    cache = make_cache(w)
    codes = {}
    for blk in range(w.NB):
        for b in range(w.B):
            for h in range(w.Hkv):
                ik = random_indices(w, layer, blk, 0, b, h, range(w.Nmax))
                iv = random_indices(w, layer, blk, 1, b, h, range(w.Nmax))
                codes[(blk, b, h)] = (ik, iv)
                words_view(cache, layer, blk, b, h).copy_(torch.from_numpy(pack_words(ik, iv, cache.NP).view(np.int32)))
    return cache, codes


def _oracle_windowed(w, codes, t, qb, kw_bits, vw_bits, nw, lo, hi, scale):
    """Per (b, hq): window tokens 0..nw[b]-1 of the bf16 arrays plus coded tokens lo[b]..hi[b]-1."""
    blk, m = t // w.Tc, t % w.Tc
    qpk = w.Hq // w.Hkv
    ref = np.zeros((w.B, w.Hq, w.D))
    lref = np.zeros((w.B, w.Hq))
    for b in range(w.B):
        for hq in range(w.Hq):
            h = hq // qpk
            ik, iv = codes[(blk, b, h)]
            a, e = int(lo[b]), max(int(hi[b]), int(lo[b]))
            kw = bf16_bits_to_f32(kw_bits[b, h, :nw[b]]) if kw_bits is not None else np.zeros((0, w.D))
            vw = bf16_bits_to_f32(vw_bits[b, h, :nw[b]]) if vw_bits is not None else np.zeros((0, w.D))
            ref[b, hq], lref[b, hq] = O.decode_windowed(
                bf16_bits_to_f32(qb[b, hq]).astype(np.float64), kw, vw, ik[a:e], iv[a:e],
                np_codebook_f32(w, 0, blk, 0, h), np_codebook_f32(w, 0, blk, 1, h), w.c, w.Tc, m, a, w.theta, scale)
    return ref, lref


@pytest.mark.parametrize("w", [CODED, CODED_GQA], ids=["mha", "gqa"])
def test_decode_range_parity(w):
    """Coded tokens start_b <= n < len_b only; starts off the 4-token tiles are masked inside the tile."""
    cache, codes = _coded_cache(w)
    starts = np.array([0, 5, 130, 7][:w.B], np.int32)
    lens = np.array([w.Nmax, 233, 131, 7][:w.B], np.int32)
    t = 2
    qb = queries(w, 0, t)
    out, lse = LQ.decode_attn_range(cache, 0, t, _dev_bits(qb), _dev_i32(starts), _dev_i32(lens), int(lens.max()))
    torch.cuda.synchronize()
    ref, lref = _oracle_windowed(w, codes, t, qb, None, None, [0] * w.B, starts, lens, 1 / math.sqrt(w.D))
    ok, msg = attn_tolerance_ok(out.cpu().numpy(), ref, lse.cpu().numpy(), lref)
    assert ok, msg


MANY = WORKLOADS["ctx4k"].replace(L=1, B=24, Hkv=2, Hq=2, Nmax=512)
MANY_GQA = WORKLOADS["gqa16k"].replace(L=1, B=20, Hkv=2, Hq=8, Nmax=256)


@pytest.mark.parametrize("w", [MANY, MANY_GQA], ids=["mha", "gqa"])
@pytest.mark.parametrize("kind", ["short", "tiny"])
def test_decode_pieces_many_segments(w, kind):
    """The split kernel shares the tiles of all (KV head, sequence) segments evenly among its CTAs: here
    CTAs run across many short segments ("short"), or outnumber the tiles so that some hold none
    ("tiny"); empty sequences, empty ranges and starts inside a tile included."""
    cache, codes = _coded_cache(w)
    rng = np.random.default_rng(23 if kind == "short" else 29)
    if kind == "short":
        lens = rng.choice([0, 1, 3, 4, 9, 37, 100, w.Nmax // 2, w.Nmax], w.B).astype(np.int32)
    else:
        lens = rng.choice([0, 1, 2, 4, 5], w.B).astype(np.int32)
    starts = np.array([rng.integers(0, int(l) + 1) for l in lens], np.int32)
    starts[:3] = 0
    t = 1
    qb = queries(w, 0, t)
    for with_starts in (False, True):
        st = starts if with_starts else np.zeros(w.B, np.int32)
        if with_starts:
            out, lse = LQ.decode_attn_range(cache, 0, t, _dev_bits(qb), _dev_i32(st), _dev_i32(lens), w.Nmax)
        else:
            out, lse = LQ.decode_attn(cache, 0, t, _dev_bits(qb), _dev_i32(lens), w.Nmax)
        torch.cuda.synchronize()
        ref, lref = _oracle_windowed(w, codes, t, qb, None, None, [0] * w.B, st, lens, 1 / math.sqrt(w.D))
        out, lse = out.cpu().numpy(), lse.cpu().numpy()
        ok, msg = attn_tolerance_ok(out, ref, lse, lref)
        assert ok, f"{kind} starts={with_starts}: {msg}"
        empty = st >= lens
        assert (out[empty] == 0).all() and np.isneginf(lse[empty]).all()


@pytest.mark.parametrize("w", [CODED, CODED_GQA], ids=["mha", "gqa"])
@pytest.mark.parametrize("t", [0, 3])
def test_windowed_cache_parity(w, t):
    """Sink tokens 0..7 and recent tokens len-64..len-1 in a bf16 window, the rest coded: bf16 kernel +
    coded range kernel + merge2 against one softmax over all tokens."""
    cache, codes = _coded_cache(w)
    lens = np.array([w.Nmax, 200, 72, 30][:w.B], np.int32)
    nw = np.minimum(lens, N_SINK + N_RECENT).astype(np.int32)        # window fill
    lo = np.minimum(lens, N_SINK).astype(np.int32)                     # coded range [lo, hi)
    hi = np.maximum(lens - N_RECENT, lo).astype(np.int32)
    W = N_SINK + N_RECENT
    kw_bits, vw_bits = _bf16_cache_bits(w, 0, t, W)
    win = LQ.Bf16Cache(_dev_bits(kw_bits), _dev_bits(vw_bits), w.Hq)
    qb = queries(w, 0, t)
    q = _dev_bits(qb)
    ow, lw = LQ.bf16_decode_attn(win, q, _dev_i32(nw), W)
    oc, lc = LQ.decode_attn_range(cache, 0, t, q, _dev_i32(lo), _dev_i32(hi), int(hi.max()))
    out, lse = LQ.merge2(oc, lc, ow, lw, out=oc, lse=lc)              # in place
    torch.cuda.synchronize()
    ref, lref = _oracle_windowed(w, codes, t, qb, kw_bits, vw_bits, nw, lo, hi, 1 / math.sqrt(w.D))
    ok, msg = attn_tolerance_ok(out.cpu().numpy(), ref, lse.cpu().numpy(), lref)
    assert ok, msg


def test_merge2_is_attention_over_the_union():
    """Two disjoint token sets attended separately (by the checker) and merged on the GPU equal one
    attention over their union; an empty part (lse = -inf) leaves the other unchanged."""
    rng = np.random.default_rng(3)
    rows, D = 6, 128
    q = rng.standard_normal((rows, D))
    parts = []
    for n in (40, 25):
        k, v = rng.standard_normal((rows, n, D)), rng.standard_normal((rows, n, D))
        parts.append((k, v))
    res = [[O.attention(q[r], k[r], v[r], 0.1) for r in range(rows)] for k, v in parts]
    oa = np.array([x[0] for x in res[0]], np.float32)
    la = np.array([x[1] for x in res[0]], np.float32)
    ob = np.array([x[0] for x in res[1]], np.float32)
    lb = np.array([x[1] for x in res[1]], np.float32)
    ob[4], lb[4] = 0.0, -np.inf                                         # row 4: part b empty
    oa[5], la[5] = 0.0, -np.inf                                         # row 5: both empty
    ob[5], lb[5] = 0.0, -np.inf
    ref, lref = [], []
    for r in range(rows):
        ka = parts[0][0][r] if r != 5 else np.zeros((0, D))
        va = parts[0][1][r] if r != 5 else np.zeros((0, D))
        kb_ = parts[1][0][r] if r < 4 else np.zeros((0, D))
        vb_ = parts[1][1][r] if r < 4 else np.zeros((0, D))
        o, l = O.attention(q[r], np.concatenate([ka, kb_]), np.concatenate([va, vb_]), 0.1)
        ref.append(o)
        lref.append(l)
    ta, tla = torch.from_numpy(oa).cuda(), torch.from_numpy(la).cuda()
    out, lse = LQ.merge2(ta, tla, torch.from_numpy(ob).cuda(), torch.from_numpy(lb).cuda(), out=ta, lse=tla)
    torch.cuda.synchronize()
    ok, msg = attn_tolerance_ok(out.cpu().numpy(), np.array(ref), lse.cpu().numpy(), np.array(lref), rel=1e-5,
                                lse_tol=1e-5)
    assert ok, msg


# ---------------------------------------------------------------- decode-time window life cycle

from synth import f32_to_bf16_bits                                    # noqa: E402
from tests.helpers import unpack_words                                 # noqa: E402

LIFE = {
    "c4tc4": WORKLOADS["ctx4k"].replace(L=2, B=2, Hkv=2, Hq=2, Nmax=128),
    "c8tc2gqa": WORKLOADS["gqa16k"].replace(L=1, T=4, Tc=2, c=8, B=2, Hkv=1, Hq=4, Nmax=128),
    "d64qpk2": WORKLOADS["tiny"].replace(B=3, Hkv=2, Hq=4, Nmax=128),
}


def _raw(w, n):
    """Pre-RoPE keys and values bits [T][B][n][Hkv][D] and keys rotated at their positions (fp64 RoPE of
    the checker, stored as bf16 like a serving cache)."""
    k = np.stack([kv_loops(w, layer, 0, 0, w.T - 1, range(w.B), range(n), range(w.Hkv)) for layer in range(w.L)])
    v = np.stack([kv_loops(w, layer, 1, 0, w.T - 1, range(w.B), range(n), range(w.Hkv)) for layer in range(w.L)])
    kf = bf16_bits_to_f32(k).astype(np.float64)                      # [L][T][B][n][Hkv][D]
    kr = np.empty_like(k)
    for idx in np.ndindex(w.L, w.T, w.B):
        for h in range(w.Hkv):
            kr[idx + (slice(None), h)] = f32_to_bf16_bits(O.rope(kf[idx + (slice(None), h)], w.theta, 0)
                                                          .astype(np.float32))
    return k, kr, v                                                   # [L][T][B][n][Hkv][D] bits


@pytest.mark.parametrize("fused", [False, True], ids=["append-then-attend", "fused"])
@pytest.mark.parametrize("name", list(LIFE))
def test_window_life_cycle(name, fused):
    """Prefill, then decode steps that roll the window twice: every attention call equals one softmax
    over the bf16 window tokens and the coded tokens, and every rolled page's codes equal the checker's
    encode of the original pre-RoPE keys and values.  "fused": the checked (layer, t) take their token
    through loopvq_window_append_decode_attn, so later calls, and the page rolls, read what its merge
    kernel wrote into the window."""
    w = LIFE[name]
    n_s, n_r = 8, 16
    P0, steps = 40, 20                                                # prefill length, decode steps
    ntot = P0 + steps
    kp, kr, vv = _raw(w, ntot)
    cache = make_cache(w)
    win = LQ.Window(cache, n_sink=n_s, n_recent=n_r)
    # ---- prefill: tokens 8 .. 23 coded, 0 .. 7 sink, 24 .. 39 recent
    coded0 = P0 - n_r
    for layer in range(w.L):
        for blk in range(w.NB):
            sl = slice(blk * w.Tc, (blk + 1) * w.Tc)
            xk = _dev_bits(kp[layer, sl, :, n_s:coded0])
            xv = _dev_bits(vv[layer, sl, :, n_s:coded0])
            LQ.encode(cache, layer, blk, xk, xv, tok0=n_s)
    order = list(range(n_s)) + list(range(coded0, P0))                # tokens in window slots 0 .. fill-1
    for dst, src in ((win.k_rot, kr), (win.k_pre, kp), (win.v, vv)):
        # [L][T][B][n][Hkv][D] -> [L][T][B][Hkv][slot][D]
        dst[:, :, :, :, :len(order)] = _dev_bits(np.ascontiguousarray(src[:, :, :, order].transpose(0, 1, 2, 4, 3, 5)))
    win.fill.fill_(len(order))
    win.coded_end.fill_(coded0)
    torch.cuda.synchronize()

    coded_end = coded0
    checks = [(0, 1), (w.L - 1, w.T - 1)]
    for step in range(steps):
        n = P0 + step                                                  # the new token
        if n_s + (n - coded_end) > n_s + n_r + 7:                      # window full: the oldest page is coded
            coded_end += 8
        LQ.window_advance(win, cache)
        for layer in range(w.L):
            for t in range(w.T):
                if not (fused and (layer, t) in checks):
                    LQ.window_append(win, layer, t, _dev_bits(kr[layer, t, :, n]), _dev_bits(kp[layer, t, :, n]),
                                     _dev_bits(vv[layer, t, :, n]))
        for layer, t in checks:
            qb = queries(w, layer, t, gain=1.0 + 0.25 * step)
            if fused:
                out, lse = LQ.window_append_decode_attn(win, cache, layer, t, _dev_bits(kr[layer, t, :, n]),
                                                        _dev_bits(kp[layer, t, :, n]), _dev_bits(vv[layer, t, :, n]),
                                                        _dev_bits(qb), w.Nmax)
            else:
                out, lse = LQ.window_decode_attn(win, cache, layer, t, _dev_bits(qb), w.Nmax)
            torch.cuda.synchronize()
            blk, m = t // w.Tc, t % w.Tc
            qpk = w.Hq // w.Hkv
            ref = np.zeros((w.B, w.Hq, w.D))
            lref = np.zeros((w.B, w.Hq))
            wtok = list(range(n_s)) + list(range(coded_end, n + 1))
            sl = slice(blk * w.Tc, (blk + 1) * w.Tc)
            for b in range(w.B):
                for h in range(w.Hkv):
                    E_k = np_codebook_f32(w, layer, blk, 0, h)
                    E_v = np_codebook_f32(w, layer, blk, 1, h)
                    ik = O.encode(bf16_bits_to_f32(kp[layer, sl, b, n_s:coded_end, h]), E_k, w.c)
                    iv = O.encode(bf16_bits_to_f32(vv[layer, sl, b, n_s:coded_end, h]), E_v, w.c)
                    for j in range(qpk):
                        hq = h * qpk + j
                        ref[b, hq], lref[b, hq] = O.decode_windowed(
                            bf16_bits_to_f32(qb[b, hq]).astype(np.float64),
                            bf16_bits_to_f32(kr[layer, t, b, wtok, h]), bf16_bits_to_f32(vv[layer, t, b, wtok, h]),
                            ik, iv, E_k, E_v, w.c, w.Tc, m, n_s, w.theta, 1 / math.sqrt(w.D))
            ok, msg = attn_tolerance_ok(out.cpu().numpy(), ref, lse.cpu().numpy(), lref)
            assert ok, f"{name} step {step} (layer {layer}, t {t}): {msg}"
    assert int(win.coded_end[0]) == coded_end and coded_end == coded0 + 16   # two rolls
    assert int(win.fill[0]) == n_s + (ntot - 1 - coded_end) + 1
    # ---- the rolled pages hold the checker's codes
    for layer in range(w.L):
        for blk in range(w.NB):
            sl = slice(blk * w.Tc, (blk + 1) * w.Tc)
            for b in range(w.B):
                for h in range(w.Hkv):
                    words = words_view(cache, layer, blk, b, h).cpu().numpy().view(np.uint32)
                    ck, cv = unpack_words(words, w.Nmax, cache.NP)
                    rk = O.encode(bf16_bits_to_f32(kp[layer, sl, b, n_s:coded_end, h]),
                                  np_codebook_f32(w, layer, blk, 0, h), w.c)
                    rv = O.encode(bf16_bits_to_f32(vv[layer, sl, b, n_s:coded_end, h]),
                                  np_codebook_f32(w, layer, blk, 1, h), w.c)
                    np.testing.assert_array_equal(ck[n_s:coded_end], rk)
                    np.testing.assert_array_equal(cv[n_s:coded_end], rv)


@pytest.mark.parametrize("name", list(LIFE))
def test_fused_append_equals_append_then_attend(name):
    """From the same window state, loopvq_window_append_decode_attn gives bit for bit the outputs of
    loopvq_window_append followed by loopvq_window_decode_attn, and leaves the same window."""
    w = LIFE[name]
    cache = make_cache(w)
    for layer in range(w.L):
        for blk in range(w.NB):
            for b in range(w.B):
                for h in range(w.Hkv):
                    ik = random_indices(w, layer, blk, 0, b, h, range(w.Nmax))
                    iv = random_indices(w, layer, blk, 1, b, h, range(w.Nmax))
                    words_view(cache, layer, blk, b, h).copy_(torch.from_numpy(pack_words(ik, iv, cache.NP).view(np.int32)))
    win = LQ.Window(cache, n_sink=8, n_recent=16)
    gen = torch.Generator(device="cuda").manual_seed(11)
    for buf in (win.k_rot, win.k_pre, win.v):
        buf.copy_(torch.randn(buf.shape, generator=gen, device="cuda").to(torch.bfloat16))
    win.fill.copy_(torch.tensor([win.W - 5, 9, win.W][:w.B], dtype=torch.int32))
    win.coded_end.copy_(torch.tensor([60, 32, 100][:w.B], dtype=torch.int32))
    new = [torch.randn((w.B, w.Hkv, w.D), generator=gen, device="cuda").to(torch.bfloat16) for _ in range(3)]
    saved = [x.clone() for x in (win.k_rot, win.k_pre, win.v)]
    for layer, t in ((0, 0), (w.L - 1, w.T - 1)):
        q = _dev_bits(queries(w, layer, t))
        for x, y in zip((win.k_rot, win.k_pre, win.v), saved):
            x.copy_(y)
        LQ.window_append(win, layer, t, *new)
        o1, l1 = LQ.window_decode_attn(win, cache, layer, t, q, w.Nmax)
        after = [x.clone() for x in (win.k_rot, win.k_pre, win.v)]
        for x, y in zip((win.k_rot, win.k_pre, win.v), saved):
            x.copy_(y)
        o2, l2 = LQ.window_append_decode_attn(win, cache, layer, t, *new, q, w.Nmax)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), (layer, t)
        for x, y in zip((win.k_rot, win.k_pre, win.v), after):
            assert torch.equal(x, y), (layer, t)
