"""The seeded input generator: Philox known answers, distribution shape, bf16 rounding."""
import json
import os

import numpy as np
import torch

from synth import (WORKLOADS, philox4x32, kv_loops, codebook, queries, lengths, random_indices,
                   f32_to_bf16_bits, bf16_bits_to_f32)


def test_philox_known_answers(golden_dir):
    with open(os.path.join(golden_dir, "philox_kat.json")) as f:
        kat = json.load(f)
    for v in kat["vectors"]:
        ctr = [int(s, 16) for s in v["ctr"]]
        key = [int(s, 16) for s in v["key"]]
        out = philox4x32(*ctr, *key)
        assert [int(o) for o in out] == [int(s, 16) for s in v["out"]]


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 37
    ours = f32_to_bf16_bits(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, theirs)
    np.testing.assert_array_equal(bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_ar1_loop_correlation_and_moments():
    w = WORKLOADS["ctx4k"]
    x = kv_loops(w, 3, 0, 0, 3, [1], range(64), range(4), dtype="f32")   # [4][1][64][4][128]
    x = x.reshape(4, -1).astype(np.float64)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02
    for t in range(1, 4):
        r = np.corrcoef(x[t - 1], x[t])[0, 1]
        assert abs(r - w.rho[t]) < 0.02


def test_slices_regenerate_identically():
    w = WORKLOADS["ctx32k"]
    full = kv_loops(w, 1, 1, 0, 3, [2, 5], range(100, 108), range(16))
    part = kv_loops(w, 1, 1, 2, 3, [5], range(104, 106), [7])
    np.testing.assert_array_equal(full[2:, 1:2, 4:6, 7:8], part)


def test_codebook_and_query_shapes():
    w = WORKLOADS["gqa16k"]
    cb = codebook(w, 0, 0, 1, 3)
    assert cb.shape == (256, 32) and cb.dtype == np.uint16
    q = queries(w, 2, 1)
    assert q.shape == (w.B, w.Hq, w.D)
    lens = lengths(WORKLOADS["ctx32k"])
    assert lens.min() >= 16384 and lens.max() <= 32768 and len(set(lens.tolist())) > 4
    assert (lengths(w) == w.Nmax).all()
    idx = random_indices(w, 0, 0, 0, 1, 2, range(10))
    assert idx.shape == (10, 16)
