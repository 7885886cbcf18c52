"""The even sharing of the coded split kernel's tiles among its CTAs, restated on the host.

The split kernel lays the 4-token tiles of every (KV head h, sequence b) segment end to end, segment
s = h * B + b, and gives CTA c of G the tiles [c T / G, (c + 1) T / G).  Each CTA writes one partial
record per segment it touches, at index s + c, and the merge of segment s reads the records of the
CTAs that hold its first through its last tile, skipping CTAs without tiles.  These tests check, for
random lengths, starts and grid sizes, that this numbering is collision-free, stays below
B * Hkv + G, and that the merge reads exactly the records the CTAs write.
"""
import numpy as np
import pytest


def seq_tiles(length, start):
    base = start & ~3
    return (length - base + 3) >> 2 if length > start else 0


def cta_first_tile(c, T, G):
    return c * T // G


def cta_of_tile(x, T, G):
    return ((x + 1) * G + T - 1) // T - 1


def written_records(lens, starts, Hkv, G):
    """(record index -> (segment, CTA, tiles)) as the CTAs write them: each walks its tile range."""
    B = len(lens)
    tiles = [seq_tiles(int(l), int(s)) for l, s in zip(lens, starts)]
    Tb = sum(tiles)
    T = Tb * Hkv
    recs = {}
    for c in range(G):
        x0, x1 = cta_first_tile(c, T, G), cta_first_tile(c + 1, T, G)
        pos = x0
        seg0 = 0
        for s in range(B * Hkv):                     # the kernel finds its first segment by a scan
            b = s % B
            seg_end = seg0 + tiles[b]
            pend = min(seg_end, x1)
            if pend > max(pos, seg0) and pos < x1:
                lo = max(pos, seg0)
                assert s + c not in recs, "two pieces share a record"
                recs[s + c] = (s, c, pend - lo)
                pos = pend
            seg0 = seg_end
    return recs, tiles, T


def merged_records(b, h, B, Hkv, tiles, T, G):
    Tb = sum(tiles)
    P = h * Tb + sum(tiles[:b])
    E = P + tiles[b]
    if E <= P:
        return []
    c0, c1 = cta_of_tile(P, T, G), cta_of_tile(E - 1, T, G)
    s = h * B + b
    return [s + c for c in range(c0, c1 + 1) if cta_first_tile(c, T, G) < cta_first_tile(c + 1, T, G)]


@pytest.mark.parametrize("seed", range(40))
def test_records_written_equal_records_merged(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 30))
    Hkv = int(rng.integers(1, 5))
    Nmax = int(rng.choice([8, 64, 300, 4096]))
    lens = rng.integers(0, Nmax + 1, B)
    if seed % 3 == 0:
        lens = rng.integers(0, 6, B)                 # fewer tiles than CTAs
    starts = np.array([rng.integers(0, int(l) + 1) for l in lens])
    G = int(rng.integers(1, 600))
    recs, tiles, T = written_records(lens, starts, Hkv, G)
    assert all(r < B * Hkv + G for r in recs)
    assert sum(n for _, _, n in recs.values()) == T   # every tile in exactly one piece
    seen = set()
    for h in range(Hkv):
        for b in range(B):
            want = merged_records(b, h, B, Hkv, tiles, T, G)
            got = sorted(r for r, (s, _, _) in recs.items() if s == h * B + b)
            assert want == got, (b, h)
            seen.update(want)
    assert seen == set(recs)


def test_shares_are_even():
    lens = np.array([18460, 28363, 24578, 16564, 31514, 21536, 21419, 26134])
    recs, tiles, T = written_records(lens, np.zeros(8, int), 16, 444)
    per_cta = {}
    for s, c, n in recs.values():
        per_cta[c] = per_cta.get(c, 0) + n
    assert max(per_cta.values()) - min(per_cta.values()) <= 1


@pytest.mark.parametrize("seed", range(20))
def test_a_cta_never_returns_to_a_kv_head(seed):
    """The one-head and four-head decode kernels keep their staged codebook tables while a CTA's next
    piece has the same KV head.  That is sound because a CTA walks its pieces in segment order, s = h B + b,
    so its heads never decrease: once it leaves a head it does not come back to it."""
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 30))
    Hkv = int(rng.integers(1, 9))
    lens = rng.integers(0, int(rng.choice([8, 300, 4096])) + 1, B)
    starts = np.array([rng.integers(0, int(l) + 1) for l in lens])
    G = int(rng.integers(1, 600))
    recs, _, _ = written_records(lens, starts, Hkv, G)
    walks = {}
    for r in sorted(recs):                               # record index s + c grows along a CTA's walk
        s, c, _ = recs[r]
        walks.setdefault(c, []).append(s // B)
    for c, heads in walks.items():
        assert heads == sorted(heads), (c, heads)


def test_ctx32k_ctas_restage_rarely():
    """At ctx32k (296 CTAs, 8 sequences, 16 KV heads) most CTAs touch one or two pieces of one head; the
    tables are staged once per head a CTA visits."""
    lens = np.array([18460, 28363, 24578, 16564, 31514, 21536, 21419, 26134])
    recs, _, _ = written_records(lens, np.zeros(8, int), 16, 296)
    pieces, heads = {}, {}
    for s, c, _ in recs.values():
        pieces[c] = pieces.get(c, 0) + 1
        heads.setdefault(c, set()).add(s // 8)
    stagings = sum(len(v) for v in heads.values())
    assert stagings < sum(pieces.values())
    assert max(len(v) for v in heads.values()) <= 2
