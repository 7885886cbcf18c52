"""The bench's roofline arithmetic, pinned to figures worked out from the definitions by hand.

ctx32k: 8 sequences of seeded lengths (18460, 28363, 24578, 16564, 31514, 21536, 21419, 26134; 188,568
tokens), 16 KV and 16 query heads, D = 128, c = 4, K = 256.  Per (layer, loop step) call:
  index words   188,568 tokens x 16 heads x 2 (K, V) x 32 one-byte codes      = 193,093,632 B
  slices        2 x 16 heads x 256 entries x 4 channels x 2 B                 =      65,536 B
  query         8 x 16 x 128 x 2 B                                             =      32,768 B
  output, lse   8 x 16 x 128 x 4 B + 8 x 16 x 4 B                              =      66,048 B
  total                                                                        = 193,257,984 B
  shared-memory gathers  188,568 x 16 x (128 + 128) x 2 B                      = 1,544,749,056 B
  fp32 work     188,568 x 16 x (3 x 128 + 4 x 128)                             = 2,703,310,848 flop
"""
import numpy as np
import pytest

import bench
from synth import WORKLOADS, lengths


def test_ctx32k_call_figures():
    w = WORKLOADS["ctx32k"]
    lens = lengths(w)
    assert int(lens.sum()) == 188568
    assert bench.call_bytes(w, lens) == 193257984
    assert bench.gather_bytes(w, lens) == 1544749056
    assert bench.call_flops(w, lens) == 2703310848


def test_ctx32k_floors_and_binding_one():
    """At 1965 MHz and the measured 6537 GB/s copy: HBM 193,257,984 B / 6537 GB/s = 29.56 us; shared memory
    1,544,749,056 B / (128 B x 148 x 1.965 GHz = 37.22 TB/s) = 41.50 us; fp32 2.703 GFLOP / (256 x 148 x
    1.965 GHz = 74.45 TFLOP/s) = 36.31 us.  The shared-memory floor binds."""
    w = WORKLOADS["ctx32k"]
    fl = bench.floors(w, lengths(w), 1965.0, 6537.0)
    assert fl["hbm"]["us"] == pytest.approx(29.5637, rel=1e-4)
    assert fl["smem"]["us"] == pytest.approx(41.4977, rel=1e-4)
    assert fl["fp32"]["us"] == pytest.approx(36.3105, rel=1e-4)
    assert max(fl, key=lambda k: fl[k]["us"]) == "smem"


def test_gqa16k_binds_on_fp32():
    """64 x 16384 tokens, 4 KV heads with 4 query heads each: 4,194,304 token-KV-heads x (3 x 128 +
    4 x 128 x 4) = 10.2 GFLOP, 137.0 us at 74.45 TFLOP/s; the gathers take 57.7 us."""
    w = WORKLOADS["gqa16k"]
    lens = lengths(w)
    assert int(lens.sum()) * w.Hkv == 4194304
    assert bench.call_flops(w, lens) == 4194304 * (3 * 128 + 4 * 128 * 4)
    fl = bench.floors(w, lens, 1965.0, 6537.0)
    assert fl["fp32"]["us"] == pytest.approx(137.01, rel=1e-3)
    assert fl["smem"]["us"] == pytest.approx(57.69, rel=1e-3)
    assert max(fl, key=lambda k: fl[k]["us"]) == "fp32"


@pytest.mark.parametrize("name", ["ctx4k", "deep32", "ctx32k_cq", "ctx32k_pg", "ctx32k_tasq"])
def test_floors_scale_with_clock_and_bandwidth(name):
    """The shared-memory and fp32 floors are inverse in the SM clock, the HBM floor in the copy bandwidth."""
    w = WORKLOADS[name]
    lens = lengths(w)
    a, b = bench.floors(w, lens, 1965.0, 6537.0), bench.floors(w, lens, 982.5, 3268.5)
    for k in ("hbm", "smem", "fp32"):
        assert b[k]["us"] == pytest.approx(2 * a[k]["us"], rel=1e-12)
    assert bench.gather_bytes(w, lens) == int(np.sum(lens)) * w.Hkv * 4 * w.D
