"""Pins of the CPU checker to facts the pages and mathematics fix.

Each test checks the checker against something that is not its own code: a
value or ratio printed on the pages (tests/golden/, each with its citation), a
closed form, an invariant, a special case that reduces to a textbook routine
(numpy / scipy), or brute force on tiny inputs.  Together they are chosen so a
dropped term, a wrong sign or index, or a transposed operand anywhere in the
checker fails one of them.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import oracle as O
from synth import WORKLOADS, kv_loops, codebook, queries, bf16_bits_to_f32, f32_to_bf16_bits

RNG = np.random.default_rng(12345)


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _rand_bf16(shape, scale=1.0):
    return bf16_bits_to_f32(f32_to_bf16_bits((RNG.standard_normal(shape) * scale).astype(np.float32)))


# ---------------------------------------------------------------- bit budget

def test_worked_example_index_count(golden_dir):
    """p2's worked example: D=128, T=4, K=256, G=16 -> 32 indices per token-head, 4 ch x 4 steps."""
    ex = _load(golden_dir, "worked_example.json")
    Tc, D, G = ex["T"], ex["D"], ex["G"]
    c = G // Tc
    assert c == ex["channels_per_chunk_per_step"] and Tc == ex["loop_steps_per_chunk"]
    x = _rand_bf16((Tc, 3, D))
    E = _rand_bf16((ex["K"], G))
    idx = O.encode(x, E, c)
    assert idx.shape == (3, ex["indices_per_token_head"])
    # per-step coding (CQ) of the same bits: D/G chunks of G channels per step, T copies
    assert ex["cq_chunks_per_step"] * ex["T"] == ex["indices_per_token_head"]
    bits = idx.shape[1] * math.log2(ex["K"]) / (Tc * D)
    assert bits == ex["bits_per_element"]


@pytest.mark.parametrize("case", range(2))
def test_bits_per_element_and_read_volume(golden_dir, case):
    """b/G bits per element; 32x / 64x below bf16; 8x / 16x fewer bytes per loop-step read."""
    cs = _load(golden_dir, "bitwidths.json")["cases"][case]
    Tc, c, D = cs["Tc"], cs["c"], cs["D"]
    x = _rand_bf16((Tc, 2, D))
    E = _rand_bf16((2 ** cs["b"], cs["G"]))
    idx = O.encode(x, E, c)
    elems_covered = Tc * D                     # one index row serves every loop step of the block
    bits = idx.shape[1] * cs["b"] / elems_covered
    assert bits == cs["bits_per_element"] == cs["b"] / cs["G"]
    assert 16 / bits == cs["compression_vs_bf16"]
    # a loop step reads the D/c index bytes of K and of V per head and token, bf16 reads 2*D*2 bytes
    assert idx.shape[1] == cs["indices_per_head_token_step"]
    assert (2 * D * 2) / (2 * idx.shape[1]) == cs["read_reduction_per_step_vs_bf16_kv"]


def test_workload_bitwidths():
    for w in WORKLOADS.values():
        want = 0.25 if w.c == 8 else 0.5
        assert 8 / w.G == want


# ---------------------------------------------------------------- encode

def test_encode_matches_brute_force_fp64():
    """Tiny inputs: every index equals the fp64 brute-force argmin, except documented near-ties."""
    Tc, N, D, c, K = 4, 40, 16, 4, 64
    x = _rand_bf16((Tc, N, D))
    E = _rand_bf16((K, c * Tc))
    idx = O.encode(x, E, c)
    # independent coupled vectors: gather loop steps on the last axis, then flatten (channel-major)
    z = x.reshape(Tc, N, D // c, c).transpose(1, 2, 3, 0).reshape(N, D // c, c * Tc).astype(np.float64)
    d = ((z[:, :, None, :] - E.astype(np.float64)[None, None, :, :]) ** 2).sum(-1)
    bf = d.argmin(-1)
    mism = idx != bf
    for n, g in zip(*np.nonzero(mism)):
        a, b = d[n, g, idx[n, g]], d[n, g, bf[n, g]]
        assert abs(a - b) <= 1e-5 * max(a, b), (n, g, a, b)
    assert mism.mean() < 0.01


def test_encode_exact_member_and_coordinate_order():
    """A codebook holding the block's own coupled vectors reconstructs them exactly (zhat = e_a(z))."""
    Tc, N, D, c = 4, 16, 16, 4
    x = _rand_bf16((Tc, N, D))
    # the coupled vector of (n, g): coordinate i*Tc + m is channel g*c+i at loop step m
    E = np.zeros((N * (D // c), c * Tc), np.float32)
    for n in range(N):
        for g in range(D // c):
            for i in range(c):
                for m in range(Tc):
                    E[n * (D // c) + g, i * Tc + m] = x[m, n, g * c + i]
    perm = RNG.permutation(E.shape[0])
    E = E[perm]
    idx = O.encode(x, E, c)
    inv = np.argsort(perm)
    for n in range(N):
        for g in range(D // c):
            assert idx[n, g] == inv[n * (D // c) + g]
            assert O.dist64(x, E, c, n, g, int(idx[n, g])) == 0.0
    for m in range(Tc):
        rec = O.dequant(idx, E, c, Tc, m)
        np.testing.assert_array_equal(rec, x[m].astype(np.float64))


def test_encode_lowest_index_on_exact_ties():
    Tc, N, D, c = 4, 5, 8, 4
    x = _rand_bf16((Tc, N, D))
    E = _rand_bf16((6, 16))
    E = np.concatenate([E, E], 0)                   # exact duplicates at r and r + 6
    idx = O.encode(x, E, c)
    assert (idx < 6).all()
    assert (O.encode(x, E[:1], c) == 0).all()        # K = 1: everything codes to entry 0


def test_encode_fp32_input_path():
    """fp32 (non-bf16) inputs: argmin still equals brute force up to near-ties."""
    Tc, N, D, c, K = 4, 30, 8, 4, 32
    x = RNG.standard_normal((Tc, N, D)).astype(np.float32)
    E = RNG.standard_normal((K, 16)).astype(np.float32)
    idx = O.encode(x, E, c)
    z = x.reshape(Tc, N, D // c, c).transpose(1, 2, 3, 0).reshape(N, D // c, 16).astype(np.float64)
    d = ((z[:, :, None, :] - E.astype(np.float64)) ** 2).sum(-1)
    bf = d.argmin(-1)
    ok = (idx == bf) | np.isclose(np.take_along_axis(d, idx[..., None].astype(np.int64), -1)[..., 0],
                                  d.min(-1), rtol=1e-5, atol=0)
    assert ok.all()


# ---------------------------------------------------------------- dequant

def test_dequant_hand_worked(golden_dir):
    g = _load(golden_dir, "dequant_hand.json")
    Tc, c, K = g["Tc"], g["c"], g["K"]
    E = np.array([[100 * r + k for k in range(c * Tc)] for r in range(K)], np.float32)
    idx = np.array(g["idx"], np.uint8)
    for m, want in g["expected_by_loop_step"].items():
        np.testing.assert_array_equal(O.dequant(idx, E, c, Tc, int(m)), np.array(want, np.float64))


def test_index_sharing_across_loop_steps():
    """Flipping one stored index changes that group's channels at all Tc loop steps and nothing else."""
    Tc, N, D, c, K = 4, 6, 32, 4, 256
    E = _rand_bf16((K, c * Tc))
    idx = RNG.integers(0, K, (N, D // c)).astype(np.uint8)
    base = [O.dequant(idx, E, c, Tc, m) for m in range(Tc)]
    n0, g0 = 3, 5
    idx2 = idx.copy()
    idx2[n0, g0] = (int(idx2[n0, g0]) + 17) % K
    for m in range(Tc):
        diff = O.dequant(idx2, E, c, Tc, m) != base[m]
        expect = np.zeros_like(diff)
        expect[n0, g0 * c:(g0 + 1) * c] = True
        # every channel of the group moves (entries differ almost surely in every coordinate)
        np.testing.assert_array_equal(diff, expect)


# ---------------------------------------------------------------- RoPE

def _rope_complex(x, pos, theta=1.0e4):
    """Textbook rotary embedding as complex rotation of (x_f + i x_{f+D/2})."""
    N, D = x.shape
    h = D // 2
    f = np.arange(h)
    ang = np.asarray(pos, np.float64)[:, None] * theta ** (-2.0 * f / D)[None, :]
    zc = (x[:, :h] + 1j * x[:, h:]) * np.exp(1j * ang)
    return np.concatenate([zc.real, zc.imag], axis=1)


def test_rope_matches_complex_rotation():
    x = RNG.standard_normal((9, 64))
    pos = np.arange(9)
    np.testing.assert_allclose(O.rope(x, 1.0e4, 0), _rope_complex(x, pos), rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.rope(x, 1.0e4, 30000), _rope_complex(x, pos + 30000), rtol=0, atol=1e-9)


def test_rope_closed_form_pair_and_identity():
    D = 8
    x = np.zeros((2, D))
    x[:, 0] = 1.0                                    # unit vector on channel 0 at positions 0 and 1
    y = O.rope(x)
    np.testing.assert_array_equal(y[0], x[0])        # position 0 is the identity
    # position 1, frequency 0 (omega = 1): only channels 0 and D/2 mix
    want = np.zeros(D)
    want[0], want[D // 2] = math.cos(1.0), math.sin(1.0)
    np.testing.assert_allclose(y[1], want, atol=1e-15)


def test_rope_relative_position_invariance():
    D = 128
    a = RNG.standard_normal((1, D))
    b = RNG.standard_normal((1, D))
    for p, j, delta in [(5, 17, 100), (0, 3000, 12345), (31000, 2, 1700)]:
        s1 = (O.rope(a, 1e4, p) * O.rope(b, 1e4, j)).sum()
        s2 = (O.rope(a, 1e4, p + delta) * O.rope(b, 1e4, j + delta)).sum()
        assert abs(s1 - s2) < 1e-11


# ---------------------------------------------------------------- attention and the split merge

def _softmax_attention_np(q, k, v, scale):
    s = k @ q * scale
    lse = logsumexp(s)
    return np.exp(s - lse) @ v, lse


def test_attention_textbook():
    q, k, v = RNG.standard_normal(16), RNG.standard_normal((50, 16)), RNG.standard_normal((50, 16))
    out, lse = O.attention(q, k, v, 0.25)
    ro, rl = _softmax_attention_np(q, k, v, 0.25)
    np.testing.assert_allclose(out, ro, rtol=1e-12, atol=1e-13)
    assert abs(lse - rl) < 1e-12


def test_attention_special_cases():
    k, v = RNG.standard_normal((33, 8)), RNG.standard_normal((33, 8))
    out, lse = O.attention(np.zeros(8), k, v, 1.0)              # q = 0 -> uniform weights
    np.testing.assert_allclose(out, v.mean(0), atol=1e-14)
    assert abs(lse - math.log(33)) < 1e-13
    out, _ = O.attention(RNG.standard_normal(8), k, np.ones_like(v), 1.0)   # all-one values
    np.testing.assert_allclose(out, np.ones(8), atol=1e-14)
    q = RNG.standard_normal(8)
    o1, l1 = O.attention(q, k, v, 0.5)
    o2, l2 = O.attention(q, k + 3.0 * q / (q @ q), v, 0.5)      # every score shifted by 1.5
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    assert abs((l2 - l1) - 1.5) < 1e-12
    out, lse = O.attention(q, np.zeros((0, 8)), np.zeros((0, 8)), 1.0)
    assert lse == -math.inf and (out == 0).all()


@pytest.mark.parametrize("bounds", [[0, 50], [0, 1, 50], [0, 7, 8, 31, 50], [0, 0, 25, 25, 50]])
def test_split_merge_is_exact(bounds):
    q, k, v = RNG.standard_normal(12), RNG.standard_normal((50, 12)), RNG.standard_normal((50, 12))
    o1, l1 = O.attention(q * 4, k, v, 0.3)
    o2, l2 = O.attention_splits(q * 4, k, v, 0.3, bounds)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    assert abs(l1 - l2) < 1e-12


# ---------------------------------------------------------------- whole decode

def _plain_rope_attention(q, kx, vx, scale, theta=1.0e4):
    kr = _rope_complex(kx, np.arange(kx.shape[0]), theta)
    return _softmax_attention_np(q, kr, vx, scale)


@pytest.mark.parametrize("m", range(4))
def test_lossless_decode_is_textbook_rope_attention(m):
    """tiny-shape block with 16 tokens x 16 groups = 256 sub-vectors used as the codebook itself:
    quantisation is lossless, so decode must equal plain RoPE attention on the original keys and values.
    Pins: keys coded before RoPE, RoPE applied to the reconstruction, per-step slice, softmax."""
    w = WORKLOADS["tiny"]
    N, D, c, Tc = 16, w.D, w.c, w.Tc
    xk = bf16_bits_to_f32(kv_loops(w, 0, 0, 0, Tc - 1, [0], range(N), [0]))[:, 0, :, 0, :]
    xv = bf16_bits_to_f32(kv_loops(w, 0, 1, 0, Tc - 1, [0], range(N), [0]))[:, 0, :, 0, :]

    def own_codebook(x):
        z = x.reshape(Tc, N, D // c, c).transpose(1, 2, 3, 0).reshape(N * D // c, c * Tc)
        return np.ascontiguousarray(z)

    Ek, Ev = own_codebook(xk), own_codebook(xv)
    ik, iv = O.encode(xk, Ek, c), O.encode(xv, Ev, c)
    q = bf16_bits_to_f32(queries(w, 0, m))[0, 0].astype(np.float64)
    scale = 1 / math.sqrt(D)
    out, lse = O.decode(q, ik, iv, Ek, Ev, c, Tc, m, 1.0e4, scale)
    ro, rl = _plain_rope_attention(q, xk[m].astype(np.float64), xv[m].astype(np.float64), scale)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    assert abs(lse - rl) < 1e-11


def test_decode_empty_cache():
    E = _rand_bf16((256, 16))
    out, lse = O.decode(np.ones(64), np.zeros((0, 16), np.uint8), np.zeros((0, 16), np.uint8), E, E, 4, 4, 0)
    assert lse == -math.inf and (out == 0).all()


def test_keys_are_rotated_values_are_not():
    """Swapping which side gets RoPE changes the answer: the checker rotates keys only."""
    w = WORKLOADS["tiny"]
    D, c, Tc, N = w.D, w.c, w.Tc, 24
    E = _rand_bf16((256, 16))
    ik = RNG.integers(0, 256, (N, D // c)).astype(np.uint8)
    iv = RNG.integers(0, 256, (N, D // c)).astype(np.uint8)
    q = RNG.standard_normal(D)
    out, lse = O.decode(q, ik, iv, E, E, c, Tc, 2, 1e4, 0.125)
    k = O.dequant(ik, E, c, Tc, 2)
    v = O.dequant(iv, E, c, Tc, 2)
    ro, rl = _softmax_attention_np(q, _rope_complex(k, np.arange(N)), v, 0.125)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    wrong, _ = _softmax_attention_np(q, k, _rope_complex(v, np.arange(N)), 0.125)
    assert np.abs(wrong - out).max() > 1e-3


# ---------------------------------------------------------------- bf16 window + coded tokens

def _window_case(NW=5, lo=9, NC=23, D=64, c=4, Tc=4, m=1):
    E_k, E_v = _rand_bf16((256, c * Tc)), _rand_bf16((256, c * Tc))
    ik = RNG.integers(0, 256, (NC, D // c)).astype(np.uint8)
    iv = RNG.integers(0, 256, (NC, D // c)).astype(np.uint8)
    kw, vw = _rand_bf16((NW, D)), _rand_bf16((NW, D))
    q = RNG.standard_normal(D)
    return q, kw, vw, ik, iv, E_k, E_v, c, Tc, m, lo


def test_windowed_is_one_softmax_over_window_and_rotated_coded_tokens():
    """Sec. 4.3 "Cache layout": window keys are taken as stored, coded keys are rebuilt and rotated at
    their absolute positions lo..hi-1; one softmax runs over all of them (numpy complex RoPE here)."""
    q, kw, vw, ik, iv, E_k, E_v, c, Tc, m, lo = _window_case()
    out, lse = O.decode_windowed(q, kw, vw, ik, iv, E_k, E_v, c, Tc, m, lo, 1e4, 0.2)
    kc = _rope_complex(O.dequant(ik, E_k, c, Tc, m), lo + np.arange(len(ik)))
    vc = O.dequant(iv, E_v, c, Tc, m)
    ro, rl = _softmax_attention_np(q, np.concatenate([kw, kc]), np.concatenate([vw, vc]), 0.2)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    assert abs(lse - rl) < 1e-11


def test_windowed_equals_merge_of_its_parts():
    """The two-kernel split of Sec. 4.3 "Attention": attention over the window alone and over the coded
    range alone, combined through their log-sum-exps (scipy), equals the windowed attention."""
    q, kw, vw, ik, iv, E_k, E_v, c, Tc, m, lo = _window_case(NW=8, lo=8, NC=40)
    out, lse = O.decode_windowed(q, kw, vw, ik, iv, E_k, E_v, c, Tc, m, lo, 1e4, 0.125)
    oa, la = O.attention(q, kw, vw, 0.125)
    ob, lb = O.decode_windowed(q, np.zeros((0, 64)), np.zeros((0, 64)), ik, iv, E_k, E_v, c, Tc, m, lo, 1e4, 0.125)
    L = logsumexp([la, lb])
    np.testing.assert_allclose(out, math.exp(la - L) * oa + math.exp(lb - L) * ob, rtol=1e-11, atol=1e-12)
    assert abs(lse - L) < 1e-11


def test_windowed_with_coded_prefix_as_window_equals_plain_decode():
    """Holding tokens 0..lo-1 in the window as their rotated reconstructions must give the same result
    as decoding all tokens from codes: pins the absolute positions of the coded part."""
    q, _, _, ik, iv, E_k, E_v, c, Tc, m, _ = _window_case(NC=30)
    lo = 6
    kw = _rope_complex(O.dequant(ik[:lo], E_k, c, Tc, m), np.arange(lo))
    vw = O.dequant(iv[:lo], E_v, c, Tc, m)
    out, lse = O.decode_windowed(q, kw, vw, ik[lo:], iv[lo:], E_k, E_v, c, Tc, m, lo, 1e4, 0.1)
    ro, rl = O.decode(q, ik, iv, E_k, E_v, c, Tc, m, 1e4, 0.1)
    np.testing.assert_allclose(out, ro, rtol=1e-10, atol=1e-12)
    assert abs(lse - rl) < 1e-10


def test_windowed_special_cases():
    q, kw, vw, ik, iv, E_k, E_v, c, Tc, m, lo = _window_case()
    z = np.zeros((0, 64))
    out, lse = O.decode_windowed(q, kw, vw, ik[:0], iv[:0], E_k, E_v, c, Tc, m, lo, 1e4, 0.3)
    ro, rl = _softmax_attention_np(q, kw, vw, 0.3)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    out, lse = O.decode_windowed(q, z, z, ik[:0], iv[:0], E_k, E_v, c, Tc, m, lo, 1e4, 0.3)
    assert lse == -math.inf and (out == 0).all()


# ---------------------------------------------------------------- one codebook per channel group

def test_pergroup_with_equal_codebooks_is_the_shared_case():
    """Every group given the same codebook: per-group encode, reconstruction and decode equal the
    shared-codebook ones (which are pinned above)."""
    D, c, Tc, N = 64, 4, 4, 20
    x = _rand_bf16((Tc, N, D))
    E = _rand_bf16((256, c * Tc))
    Eg = np.broadcast_to(E, (D // c, 256, c * Tc)).copy()
    ik = O.encode_pg(x, Eg, c)
    np.testing.assert_array_equal(ik, O.encode(x, E, c))
    np.testing.assert_array_equal(O.dequant_pg(ik, Eg, c, Tc, 2), O.dequant(ik, E, c, Tc, 2))
    q = RNG.standard_normal(D)
    o1, l1 = O.decode_pg(q, ik, ik[::-1].copy(), Eg, Eg, c, Tc, 1, 1e4, 0.2)
    o2, l2 = O.decode(q, ik, ik[::-1].copy(), E, E, c, Tc, 1, 1e4, 0.2)
    np.testing.assert_array_equal(o1, o2)
    assert l1 == l2


def test_pergroup_encode_is_brute_force_per_group():
    """Each group's index is the fp64 nearest entry of that group's own codebook."""
    D, c, Tc, N, K = 32, 8, 2, 6, 40
    x = _rand_bf16((Tc, N, D))
    Eg = _rand_bf16((D // c, K, c * Tc))
    idx = O.encode_pg(x, Eg, c)
    for n in range(N):
        for g in range(D // c):
            z = np.array([x[m, n, g * c + i] for i in range(c) for m in range(Tc)], np.float64)
            d = ((Eg[g].astype(np.float64) - z) ** 2).sum(1)
            assert idx[n, g] == int(np.argmin(d)), (n, g)
            assert abs(O.dist64_pg(x, Eg, c, n, g, int(idx[n, g])) - d.min()) < 1e-9


def test_pergroup_reconstruction_uses_only_its_group():
    """Changing group g's codebook changes exactly channels g*c .. g*c+c-1 of the reconstruction."""
    D, c, Tc, N = 64, 4, 4, 8
    Eg = _rand_bf16((D // c, 256, c * Tc))
    idx = RNG.integers(0, 256, (N, D // c)).astype(np.uint8)
    base = O.dequant_pg(idx, Eg, c, Tc, 3)
    E2 = Eg.copy()
    E2[5] += 1.0
    diff = np.abs(O.dequant_pg(idx, E2, c, Tc, 3) - base) > 0
    assert diff[:, 5 * c:6 * c].all() and not diff[:, :5 * c].any() and not diff[:, 6 * c:].any()


def test_pergroup_lossless_decode_is_textbook_rope_attention():
    """Each group's codebook holds that group's own coupled vectors: reconstruction is exact, so decode
    equals plain RoPE attention on the original keys and values (numpy complex RoPE)."""
    D, c, Tc, N, m = 64, 4, 4, 24, 2
    xk, xv = _rand_bf16((Tc, N, D)), _rand_bf16((Tc, N, D))

    def own(x):                                           # [D/c][K=N][G]: group g's vectors of all tokens
        return np.ascontiguousarray(x.reshape(Tc, N, D // c, c).transpose(2, 1, 3, 0).reshape(D // c, N, c * Tc))

    Ek, Ev = own(xk), own(xv)
    ik, iv = O.encode_pg(xk, Ek, c), O.encode_pg(xv, Ev, c)
    np.testing.assert_array_equal(ik, np.tile(np.arange(N)[:, None], (1, D // c)))
    q = RNG.standard_normal(D)
    out, lse = O.decode_pg(q, ik, iv, Ek, Ev, c, Tc, m, 1e4, 0.15)
    ro, rl = _softmax_attention_np(q, _rope_complex(xk[m].astype(np.float64), np.arange(N)),
                                   xv[m].astype(np.float64), 0.15)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    assert abs(lse - rl) < 1e-11


# ---------------------------------------------------------------- TaSQ before loop-axis coupling

def test_round_fp16_matches_the_ieee_half_conversion():
    """The checker's fp16 rounding equals numpy's float16 cast (IEEE binary16, ties to even) across
    normal, subnormal, tie, boundary and overflow values."""
    vals = np.concatenate([RNG.standard_normal(20000) * 10.0 ** RNG.integers(-9, 6, 20000),
                           np.array([0.0, 1.0, 65504.0, 65519.99, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -25,
                                     2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, -6e-5])])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).astype(np.float64)
    got = np.array([O.round_fp16(v) for v in vals])
    np.testing.assert_array_equal(got, ref)


def _tasq_case(Hkv=3, N=10, D=64, Tc=4, c=4, seed=5):
    rng = np.random.default_rng(seed)
    k = _rand_bf16((Tc, Hkv, N, D))
    wh = np.exp(rng.uniform(-0.5, 0.5, (Tc, Hkv, D // 2))).astype(np.float32)
    w = np.concatenate([wh, wh], axis=2)                  # a RoPE pair shares its weight
    perm = rng.permutation(D // 2).astype(np.int16)
    return k, w, perm


def test_tasq_sigma_is_the_rms_over_heads_and_channels_in_fp16():
    k, w, _ = _tasq_case()
    for m in range(k.shape[0]):
        sig = O.tasq_sigma(k[m], w[m])
        wk = w[m][:, None, :].astype(np.float64) * k[m].astype(np.float64)
        ref = np.sqrt((wk ** 2).mean(axis=(0, 2))).astype(np.float16).astype(np.float64)
        np.testing.assert_array_equal(sig, ref)


def test_tasq_scale_equivariance():
    """Doubling a token's keys doubles its sigma exactly and leaves u, hence its codes, unchanged."""
    k, w, perm = _tasq_case(Hkv=1, N=6)
    E = _rand_bf16((256, 16))
    sig = np.stack([O.tasq_sigma(k[m], w[m]) for m in range(4)])
    idx = O.tasq_encode(k[:, 0], w[:, 0], sig, perm, E, 4)
    k2 = k.copy()
    k2[:, :, 3] *= 2.0
    sig2 = np.stack([O.tasq_sigma(k2[m], w[m]) for m in range(4)])
    np.testing.assert_array_equal(sig2[:, 3], 2 * sig[:, 3])
    np.testing.assert_array_equal(O.tasq_encode(k2[:, 0], w[:, 0], sig2, perm, E, 4), idx)


@pytest.mark.parametrize("m", [0, 3])
def test_tasq_lossless_decode_is_textbook_rope_attention(m):
    """Codebooks holding the exact transformed coupled vectors: reconstruction inverts the weighting,
    the scale and the permutation, so decode equals plain RoPE attention on the original keys (numpy
    complex RoPE) up to the fp32 rounding of u."""
    Tc, N, D, c = 4, 16, 64, 4
    k, w, perm = _tasq_case(Hkv=1, N=N, D=D, Tc=Tc, c=c)
    k, w = k[:, 0], w[:, 0]                                # one head: [Tc][N][D], [Tc][D]
    sig = np.stack([O.tasq_sigma(k[mm][None], w[mm][None]) for mm in range(Tc)])
    u = np.stack([O.tasq_transform(k[mm], w[mm], sig[mm]) for mm in range(Tc)])   # [Tc][N][D]
    # group g of the permutation: pairs perm[g*c/2 + j] -> channels (f, f + D/2); coordinate i*Tc + mm
    ch = np.array([[perm[g * (c // 2) + i // 2] + (D // 2) * (i % 2) for i in range(c)] for g in range(D // c)])
    E = np.stack([u[:, n, ch[g]].T.reshape(-1) for n in range(N) for g in range(D // c)]).astype(np.float32)
    idx = O.tasq_encode(k, w, sig, perm, E, c)
    np.testing.assert_array_equal(idx, np.arange(N * (D // c)).reshape(N, D // c) % 256)
    kh = O.tasq_dequant(idx, E, c, Tc, m, perm, w[m], sig[m])
    np.testing.assert_allclose(kh, k[m].astype(np.float64), rtol=2e-7, atol=0)
    v = _rand_bf16((Tc, N, D))
    Ev = np.stack([np.array([v[mm, n, g * c + i] for i in range(c) for mm in range(Tc)])
                   for n in range(N) for g in range(D // c)]).astype(np.float32)
    iv = O.encode(v, Ev, c)
    q = RNG.standard_normal(D)
    out, lse = O.tasq_decode(q, idx, iv, E, Ev, perm, w[m], sig[m], c, Tc, m, 1e4, 0.2)
    ro, rl = _softmax_attention_np(q, _rope_complex(k[m].astype(np.float64), np.arange(N)),
                                   v[m].astype(np.float64), 0.2)
    np.testing.assert_allclose(out, ro, rtol=1e-6, atol=1e-7)
    assert abs(lse - rl) < 1e-6
