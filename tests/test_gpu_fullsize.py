"""Full-size workloads in the launch configuration the benchmark times, checked row by row.

A cache of one layer has exactly the per-call launch configuration of every layer
of the full model (grid and splits depend on batch, heads, head size, code width
and max length only), so each workload runs at its full batch, head count and
context.  Every (sequence, query head) row of one decode call is compared with the
checker, so every piece boundary the tile plan creates at full size is crossed.
Bulk inputs come from the CUDA generator; the checker regenerates the inputs of
each row on the CPU from the same counters.  The checker's calls run on host
threads (its ctypes calls release the GIL).  Encode checks cover every token of two
(sequence, KV head) pairs of the deep32 and ctx32k launches; the near-ties found
(codes that differ with fp64 distances within 1e-5 relative) are printed, and written to
near_ties.json in the directory LOOPVQ_RECORD_DIR names, when it is set.
"""
import json
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import looped_lm_decode_b200 as LQ
from oracle import oracle as O
from synth import WORKLOADS, lengths, random_indices, queries, kv_loops, bf16_bits_to_f32
from synth import gpu as SG
from tests.helpers import unpack_words, words_view, np_codebook_f32, attn_tolerance_ok

pytestmark = pytest.mark.gpu

THREADS = max(1, len(os.sched_getaffinity(0)))
SAMPLES = {"ctx32k": [(0, 0), (3, 7), (7, 15)], "ctx4k": [(0, 0), (31, 15)], "gqa16k": [(0, 0), (63, 13)],
           "deep32": [(1, 39), (0, 17)], "ctx32k_cq": [(0, 0), (6, 11)], "ctx32k_pg": [(2, 3), (7, 15)]}


def _record_ties(key, value):
    out = os.environ.get("LOOPVQ_RECORD_DIR", "")
    if not out or not os.path.isdir(out):
        return
    path = os.path.join(out, "near_ties.json")
    data = {}
    if os.path.exists(path):
        with open(path) as f:
            data = json.load(f)
    data[key] = value
    with open(path, "w") as f:
        json.dump(data, f, indent=1)


def _full_cache(w):
    cache = LQ.Cache(w.L, w.T, w.Tc, w.Hkv, w.Hq, w.D, w.c, w.K, w.B, w.Nmax, w.theta, ncb=w.ncb)
    SG.fill_codebook(w, cache.codebook)
    LQ.prepare(cache)
    return cache


@pytest.mark.parametrize("name", list(SAMPLES))
def test_decode_full_size_every_row(name):
    w = WORKLOADS[name].replace(L=1)
    cache = _full_cache(w)
    t = w.T - 2                        # a loop step that is not the first of its block
    blk, m = t // w.Tc, t % w.Tc
    per_lb = w.B * w.Hkv * w.Nmax * cache.NP
    SG.fill_idx(w, 0, blk, cache.idx[blk * per_lb:(blk + 1) * per_lb])
    lens = lengths(w)
    qd = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    SG.fill_q(w, 0, t, qd)
    out, lse = LQ.decode_attn(cache, 0, t, qd.view(torch.int16), torch.from_numpy(lens).cuda(), int(lens.max()))
    torch.cuda.synchronize()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qpk = w.Hq // w.Hkv
    qall = queries(w, 0, t)
    cbs = {(kv, h): np_codebook_f32(w, 0, blk, kv, h) for kv in range(2) for h in range(w.Hkv)}
    dec = O.decode_pg if w.ncb > 1 else O.decode

    def row(bh):
        b, h = bh
        n = int(lens[b])
        ik = random_indices(w, 0, blk, 0, b, h, range(n))
        iv = random_indices(w, 0, blk, 1, b, h, range(n))
        res = []
        for j in range(qpk):
            hq = h * qpk + j
            res.append((b, hq) + dec(bf16_bits_to_f32(qall[b, hq]).astype(np.float64), ik, iv, cbs[(0, h)],
                                     cbs[(1, h)], w.c, w.Tc, m, w.theta, 1 / math.sqrt(w.D)))
        return res

    ref = np.zeros(out.shape)
    lref = np.zeros(lse.shape)
    with ThreadPoolExecutor(THREADS) as ex:
        for res in ex.map(row, [(b, h) for b in range(w.B) for h in range(w.Hkv)]):
            for b, hq, r, lr in res:
                ref[b, hq], lref[b, hq] = r, lr
    ok, msg = attn_tolerance_ok(out, ref, lse, lref)
    print(f"{name}: all {w.B * w.Hq} rows, {int(lens.sum())} tokens x {w.Hkv} heads: {msg}")
    assert ok, f"{name}: {msg}"
    # and row by row, against each row's own scale
    for b, hq in SAMPLES[name]:
        okr, msgr = attn_tolerance_ok(out[b, hq], ref[b, hq], lse[b, hq:hq + 1], lref[b, hq:hq + 1])
        assert okr, f"{name} (b={b}, hq={hq}): {msgr}"


def _encode_every_token(name, blk, pairs):
    """One full-size (layer, block) encode of the workload's whole batch, keys and values; every token of
    the given (sequence, KV head) pairs checked against the checker.  Returns the near-tie count."""
    w = WORKLOADS[name].replace(L=1)
    cache = _full_cache(w)
    xs = []
    for kv in range(2):
        x = torch.empty((w.Tc, w.B, w.Nmax, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
        SG.fill_kv(w, 0, kv, blk * w.Tc, blk * w.Tc + w.Tc - 1, x)
        xs.append(x)
    LQ.encode(cache, 0, blk, xs[0], xs[1])
    LQ.fault_check()
    del xs
    chunk = 1024
    gpu_codes = {}
    for b, h in pairs:
        words = words_view(cache, 0, blk, b, h).cpu().numpy().view(np.uint32)
        gpu_codes[(b, h)] = unpack_words(words, w.Nmax, cache.NP)

    def job(arg):
        b, h, kv, n0 = arg
        codes = gpu_codes[(b, h)][kv][n0:n0 + chunk]
        toks = range(n0, min(n0 + chunk, w.Nmax))
        x = kv_loops(w, 0, kv, blk * w.Tc, blk * w.Tc + w.Tc - 1, [b], toks, [h])[:, 0, :, 0, :]
        xf = np.ascontiguousarray(bf16_bits_to_f32(x))
        E = np_codebook_f32(w, 0, blk, kv, h)
        ref = O.encode(xf, E, w.c)
        ties = 0
        for i, g in zip(*np.nonzero(codes != ref)):
            dg = O.dist64(xf, E, w.c, int(i), int(g), int(codes[i, g]))
            do = O.dist64(xf, E, w.c, int(i), int(g), int(ref[i, g]))
            assert abs(dg - do) <= 1e-5 * max(dg, do), (name, b, h, kv, n0 + int(i), int(g))
            ties += 1
        return ties

    jobs = [(b, h, kv, n0) for b, h in pairs for kv in range(2) for n0 in range(0, w.Nmax, chunk)]
    with ThreadPoolExecutor(THREADS) as ex:
        ties = sum(ex.map(job, jobs))
    n_codes = len(pairs) * 2 * w.Nmax * (w.D // w.c)
    print(f"{name} encode: {n_codes} codes checked, near-ties: {ties}")
    _record_ties(f"encode_{name}", {"codes_checked": n_codes, "near_ties": ties, "pairs": pairs, "block": blk})
    return ties


def test_encode_full_size_deep32():
    """deep32 prefill encode of one (layer, block) at full size: 2 x 8192 tokens x 40 heads, K and V;
    every token of two (sequence, KV head) pairs checked."""
    _encode_every_token("deep32", 3, [(0, 0), (1, 39)])


def test_encode_full_size_ctx32k():
    """The ctx32k-shaped encode the benchmark times (8 x 32768 tokens x 16 heads, K and V); every token of
    two (sequence, KV head) pairs checked."""
    _encode_every_token("ctx32k", 0, [(0, 0), (7, 15)])


@pytest.mark.parametrize("name", ["ctx32k", "gqa16k"])
def test_bf16_cache_full_size_sampled(name):
    """The bf16-cache comparison at full size, built as bench.py builds it (loop step 1 of layer 0 as
    rotated keys / values, [B][Hkv][Nmax][D]); sampled (sequence, query head) outputs vs the checker."""
    w = WORKLOADS[name].replace(L=1)
    tmp = torch.empty((1, w.B, w.Nmax, w.Hkv, w.D), dtype=torch.bfloat16, device="cuda")
    kv = []
    for k in range(2):
        SG.fill_kv(w, 0, k, 1, 1, tmp)
        kv.append(tmp[0].permute(0, 2, 1, 3).contiguous())
    del tmp
    cache = LQ.Bf16Cache(kv[0], kv[1], w.Hq)
    lens = lengths(w)
    t = 2
    qd = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    SG.fill_q(w, 0, t, qd)
    out, lse = LQ.bf16_decode_attn(cache, qd, torch.from_numpy(lens).cuda(), int(lens.max()))
    torch.cuda.synchronize()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qpk = w.Hq // w.Hkv
    for b, hq in SAMPLES[name]:
        h = hq // qpk
        n = int(lens[b])
        kb = bf16_bits_to_f32(kv_loops(w, 0, 0, 1, 1, [b], range(n), [h])[0, 0, :, 0, :])
        vb = bf16_bits_to_f32(kv_loops(w, 0, 1, 1, 1, [b], range(n), [h])[0, 0, :, 0, :])
        qb = queries(w, 0, t, b=[b], hq=[hq])[0, 0]
        ref, lref = O.attention(bf16_bits_to_f32(qb).astype(np.float64), kb, vb, 1 / math.sqrt(w.D))
        ok, msg = attn_tolerance_ok(out[b, hq], ref, lse[b, hq:hq + 1], np.array([lref]))
        assert ok, f"{name} (b={b}, hq={hq}): {msg}"


def test_tasq_decode_full_size_sampled():
    """TaSQ keys at the full ctx32k shape in the launch configuration the benchmark times (long per-warp
    runs, so the rotation recurrence is set from the table several times); uniform random codes, seeded
    token scales, sampled (sequence, query head) outputs against the checker."""
    from synth import tasq_weights, tasq_perm
    w = WORKLOADS["ctx32k_tasq"].replace(L=1)
    cache = _full_cache(w)
    tw, tp = tasq_weights(w), tasq_perm(w)
    tq = LQ.Tasq(cache, w=torch.from_numpy(tw).cuda(), perm=torch.from_numpy(tp).cuda())
    t = 1
    blk, m = t // w.Tc, t % w.Tc
    per_lb = w.B * w.Hkv * w.Nmax * cache.NP
    SG.fill_idx(w, 0, blk, cache.idx[blk * per_lb:(blk + 1) * per_lb])
    sig = np.random.default_rng(41).uniform(0.25, 4.0, (w.L, w.T, w.B, w.Nmax)).astype(np.float16)
    tq.sigma.copy_(torch.from_numpy(sig.reshape(-1)).cuda())
    lens = lengths(w)
    qd = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    SG.fill_q(w, 0, t, qd)
    out, lse = LQ.tasq_decode_attn(cache, tq, 0, t, qd.view(torch.int16), torch.from_numpy(lens).cuda(),
                                   int(lens.max()))
    torch.cuda.synchronize()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b, hq in [(0, 0), (5, 9)]:
        h = hq
        n = int(lens[b])
        ik = random_indices(w, 0, blk, 0, b, h, range(n))
        it = np.empty_like(ik)                       # word bytes 0/1 of pair-group p: TaSQ groups 2p, 2p+1
        it[:, 0::2] = ik[:, :cache.NP]
        it[:, 1::2] = ik[:, cache.NP:]
        iv = random_indices(w, 0, blk, 1, b, h, range(n))
        qb = queries(w, 0, t, b=[b], hq=[hq])[0, 0]
        ref, lref = O.tasq_decode(bf16_bits_to_f32(qb).astype(np.float64), it, iv, np_codebook_f32(w, 0, blk, 0, h),
                                  np_codebook_f32(w, 0, blk, 1, h), tp[0, blk, h], tw[0, t, h],
                                  sig[0, t, b, :n].astype(np.float64), w.c, w.Tc, m, w.theta, 1 / math.sqrt(w.D))
        ok, msg = attn_tolerance_ok(out[b, hq], ref, lse[b, hq:hq + 1], np.array([lref]))
        print(f"ctx32k_tasq (b={b}, hq={hq}, {n} tokens): {msg}")
        assert ok, f"ctx32k_tasq (b={b}, hq={hq}): {msg}"
