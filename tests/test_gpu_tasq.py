"""TaSQ before loop-axis coupling (LoopVQ paper, App. B) on the GPU vs the CPU checker.

Encode: the fp16 token scales and every code are compared bit for bit with the checker's
(the GPU and the checker form u = (w * k) / sigma with the same fp32 roundings).  Decode: codes and
scales drawn by the test (uniform codes, fp16 scales), so no GPU output reaches the checker;
attention within max|out - ref| <= 2e-3 * ||ref||_inf, |lse - lse_ref| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import looped_lm_decode_b200 as LQ
from oracle import oracle as O
from synth import WORKLOADS, kv_loops, queries, random_indices, tasq_weights, tasq_perm, bf16_bits_to_f32
from tests.helpers import pack_words, unpack_words, words_view, make_cache, np_codebook_f32, attn_tolerance_ok

pytestmark = pytest.mark.gpu

SHAPES = {
    "c4": WORKLOADS["ctx4k"].replace(L=1, B=2, Hkv=2, Hq=2, Nmax=128),
    "c4tc2": WORKLOADS["ctx4k"].replace(L=1, Tc=2, B=2, Hkv=3, Hq=3, Nmax=64),
    "c8gqa": WORKLOADS["gqa16k"].replace(L=1, B=2, Hkv=1, Hq=4, Nmax=128),
    "c8d64": WORKLOADS["tiny"].replace(c=8, B=2, Hkv=2, Hq=2, Nmax=64),
}


def _tasq(w, cache):
    tw, tp = tasq_weights(w), tasq_perm(w)
    return LQ.Tasq(cache, w=torch.from_numpy(tw).cuda(), perm=torch.from_numpy(tp).cuda()), tw, tp


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)


def _tasq_codes(ck, NP):
    """Word bytes 0/1 of pair-group p are TaSQ groups 2p and 2p+1: back to TaSQ group order."""
    ct = np.empty_like(ck)
    ct[:, 0::2] = ck[:, :NP]
    ct[:, 1::2] = ck[:, NP:]
    return ct


@pytest.mark.parametrize("name", list(SHAPES))
def test_tasq_encode_parity(name):
    """Codes bit-exact except near-ties (fp64 distances within 1e-5 relative, counted); scales bit-exact.
    bf16 input at these shapes runs the tensor-core encode with the three-part split of u."""
    w = SHAPES[name]
    cache = make_cache(w)
    tq, tw, tp = _tasq(w, cache)
    NP = cache.NP
    ties = 0
    for blk in range(w.NB):
        x = [kv_loops(w, 0, kv, blk * w.Tc, blk * w.Tc + w.Tc - 1, range(w.B), range(w.Nmax), range(w.Hkv))
             for kv in range(2)]                                          # [Tc][B][N][Hkv][D] bits
        LQ.tasq_encode(cache, tq, 0, blk, _dev(x[0]), _dev(x[1]))
        torch.cuda.synchronize()
        sig_gpu = tq.sigma.view(w.L, w.T, w.B, w.Nmax).cpu().numpy().astype(np.float64)
        xk, xv = bf16_bits_to_f32(x[0]), bf16_bits_to_f32(x[1])
        for b in range(w.B):
            sig = np.stack([O.tasq_sigma(xk[m, b].transpose(1, 0, 2), tw[0, blk * w.Tc + m]) for m in range(w.Tc)])
            np.testing.assert_array_equal(sig_gpu[0, blk * w.Tc:(blk + 1) * w.Tc, b], sig)
            for h in range(w.Hkv):
                words = words_view(cache, 0, blk, b, h).cpu().numpy().view(np.uint32)
                ck, cv = unpack_words(words, w.Nmax, NP)
                Ek, Ev = np_codebook_f32(w, 0, blk, 0, h), np_codebook_f32(w, 0, blk, 1, h)
                rk = O.tasq_encode(xk[:, b, :, h, :], tw[0, blk * w.Tc:(blk + 1) * w.Tc, h], sig, tp[0, blk, h], Ek,
                                   w.c)
                gk = _tasq_codes(ck, NP)
                mism = np.argwhere(gk != rk)
                if len(mism):
                    # the coupled vectors of TaSQ groups: u at the permuted channels, group g = channels g c ..
                    u = np.stack([O.tasq_transform(xk[m, b, :, h, :], tw[0, blk * w.Tc + m, h], sig[m])
                                  for m in range(w.Tc)])
                    pairs = tp[0, blk, h].astype(np.int64) & (w.D // 2 - 1)
                    chans = np.stack([pairs, pairs + w.D // 2], axis=1).reshape(-1)     # (f, f + D/2) per pair
                    ut = np.ascontiguousarray(u[:, :, chans])
                    for n, g in mism:
                        dg = O.dist64(ut, Ek, w.c, n, g, int(gk[n, g]))
                        do = O.dist64(ut, Ek, w.c, n, g, int(rk[n, g]))
                        assert abs(dg - do) <= 1e-5 * max(dg, do), (b, h, n, g, dg, do)
                    ties += len(mism)
                rv = O.encode(xv[:, b, :, h, :], Ev, w.c)
                for n, g in np.argwhere(cv != rv):
                    dg = O.dist64(xv[:, b, :, h, :], Ev, w.c, n, g, int(cv[n, g]))
                    do = O.dist64(xv[:, b, :, h, :], Ev, w.c, n, g, int(rv[n, g]))
                    assert abs(dg - do) <= 1e-5 * max(dg, do), (b, h, n, g, dg, do)
                    ties += 1
    print(f"{name}: near-ties {ties}")


@pytest.mark.parametrize("name", list(SHAPES))
def test_tasq_decode_parity(name):
    w = SHAPES[name]
    cache = make_cache(w)
    tq, tw, tp = _tasq(w, cache)
    NP = cache.NP
    rng = np.random.default_rng(17)
    codes = {}
    for blk in range(w.NB):
        for b in range(w.B):
            for h in range(w.Hkv):
                it = random_indices(w, 0, blk, 0, b, h, range(w.Nmax))       # TaSQ group order
                iv = random_indices(w, 0, blk, 1, b, h, range(w.Nmax))
                codes[(blk, b, h)] = (it, iv)
                ik = np.concatenate([it[:, 0::2], it[:, 1::2]], axis=1)      # word layout: (2p, 2p+1) -> (p, p+NP)
                words_view(cache, 0, blk, b, h).copy_(torch.from_numpy(pack_words(ik, iv, NP).view(np.int32)))
    sig = rng.uniform(0.25, 4.0, (w.L, w.T, w.B, w.Nmax)).astype(np.float16)
    tq.sigma.copy_(torch.from_numpy(sig.reshape(-1)).cuda())
    lens = np.array([w.Nmax, max(1, w.Nmax // 2 - 3)], np.int32)[:w.B]
    for t in range(w.T):
        blk, m = t // w.Tc, t % w.Tc
        qb = queries(w, 0, t)
        out, lse = LQ.tasq_decode_attn(cache, tq, 0, t, _dev(qb), torch.from_numpy(lens).cuda(), int(lens.max()))
        torch.cuda.synchronize()
        qpk = w.Hq // w.Hkv
        ref = np.zeros((w.B, w.Hq, w.D))
        lref = np.zeros((w.B, w.Hq))
        for b in range(w.B):
            n = int(lens[b])
            for hq in range(w.Hq):
                h = hq // qpk
                it, iv = codes[(blk, b, h)]
                ref[b, hq], lref[b, hq] = O.tasq_decode(
                    bf16_bits_to_f32(qb[b, hq]).astype(np.float64), it[:n], iv[:n], np_codebook_f32(w, 0, blk, 0, h),
                    np_codebook_f32(w, 0, blk, 1, h), tp[0, blk, h], tw[0, t, h], sig[0, t, b, :n].astype(np.float64),
                    w.c, w.Tc, m, w.theta, 1 / math.sqrt(w.D))
        ok, msg = attn_tolerance_ok(out.cpu().numpy(), ref, lse.cpu().numpy(), lref)
        assert ok, f"{name} t {t}: {msg}"
