"""The bench's encode tie count: codes equal to the checker's count as checked with no mismatch, a code
moved to a far entry counts as one mismatch, and the sample's GPU codes are taken from a snapshot (not
re-read from a cache that a later run may have changed)."""
import numpy as np

import bench
from oracle import oracle as O
from synth import WORKLOADS, bf16_bits_to_f32, kv_loops


def _checker_codes(w, threads):
    chunk, sample = bench.tie_sample(w, threads)
    codes, inputs = {}, {}
    for b, h, tok0 in sample:
        pair = []
        for kv in range(2):
            x = kv_loops(w, 0, kv, 0, w.Tc - 1, [b], range(tok0, tok0 + chunk), [h])[:, 0, :, 0, :]
            xf = np.ascontiguousarray(bf16_bits_to_f32(x))
            E = np.ascontiguousarray(bf16_bits_to_f32(bench._codebook(w, 0, 0, kv, h)))
            pair.append(O.encode(xf, E, w.c))
            inputs[(b, h, tok0, kv)] = (xf, E)
        codes[(b, h, tok0)] = tuple(pair)
    return chunk, codes, inputs


def test_tie_count_exact_and_planted_mismatch():
    w = WORKLOADS["tiny"].replace(B=2, Hkv=2, Hq=2, Nmax=64)
    threads = 2
    chunk, codes, inputs = _checker_codes(w, threads)
    _, ties = bench.cpu_encode_and_ties(w, codes, threads, 1.0)
    assert ties["checked"] == threads * 2 * chunk * (w.D // w.c)
    assert ties["near_ties"] == 0 and ties["mismatches"] == 0

    # move one value code of the first sampled run to the entry farthest from its vector
    key = next(iter(codes))
    ck, cv = (c.copy() for c in codes[key])
    xf, E = inputs[key + (1,)]
    i, g = 3, 5
    far = max(range(w.K), key=lambda r: O.dist64(xf, E, w.c, i, g, r))
    assert far != cv[i, g]
    cv[i, g] = far
    planted = dict(codes)
    planted[key] = (ck, cv)
    _, ties = bench.cpu_encode_and_ties(w, planted, threads, 1.0)
    assert ties["near_ties"] == 0 and ties["mismatches"] == 1


def test_tie_sample_stays_inside_the_cache():
    for name in ("tiny", "ctx32k", "deep32"):
        w = WORKLOADS[name]
        for threads in (1, 16, 64):
            chunk, sample = bench.tie_sample(w, threads)
            assert len(sample) == threads
            for b, h, tok0 in sample:
                assert 0 <= b < w.B and 0 <= h < w.Hkv and 0 <= tok0 and tok0 + chunk <= w.Nmax
