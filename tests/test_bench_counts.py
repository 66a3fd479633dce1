"""bench.py's work counts against brute force over the oracle's visibility
mask: the unmasked pairs behind every effective-FLOP figure, the sampled
rows' pairs behind the oracle baseline, and the visited tile pairs behind
the ALiBi gradient's byte count.  The FLOP convention itself (forward
4 d P, backward 10 d P, counting the recompute of S) is bench.py's; here
P and its use in the closed forms are checked."""
import numpy as np
import pytest

import bench
from oracle import visibility_mask

MASKS = [
    (1, False, -1, -1), (1, True, -1, -1), (37, True, -1, -1), (130, False, -1, -1),
    (300, True, -1, -1), (300, True, 0, -1), (300, True, 100, -1), (333, False, 100, 50),
    (257, False, -1, 0), (520, True, 4096, -1), (260, False, 0, 0), (1024, True, 128, -1),
]


@pytest.mark.parametrize("L,causal,wl,wr", MASKS)
def test_visible_pairs_equal_the_mask_count(L, causal, wl, wr):
    m = visibility_mask(L, causal, wl, wr)
    assert bench.visible_pairs(L, causal, wl, wr) == int(m.sum())
    c = dict(L=L, causal=causal, wl=wl, wr=wr)
    assert bench.sample_pairs(c, None) == int(m.sum())
    rows = np.arange(0, L, 7)
    assert bench.sample_pairs(c, rows) == int(m[rows].sum())


@pytest.mark.parametrize("L,causal,wl,wr", MASKS)
def test_visited_tile_pairs_equal_the_tiles_holding_a_visible_pair(L, causal, wl, wr):
    m = visibility_mask(L, causal, wl, wr)
    n = (L + 127) // 128
    want = sum(bool(m[a * 128:(a + 1) * 128, b * 128:(b + 1) * 128].any())
               for a in range(n) for b in range(n))
    assert bench.visited_tile_pairs(dict(L=L, causal=causal, wl=wl, wr=wr)) == want


def test_benchmark_workloads_count_the_closed_forms():
    # causal L: L (L + 1) / 2 pairs per head; bidirectional: L^2; a causal
    # window w >= L - 1 changes nothing
    m4 = bench.CONFIGS["mistral4k"]
    L = m4["L"]
    assert bench.flop_counts(m4)["P"] == L * (L + 1) // 2
    t5 = bench.CONFIGS["t5rpe"]
    fl = bench.flop_counts(t5)
    assert fl["P"] == t5["L"] ** 2
    heads = t5["B"] * t5["Hq"]
    assert fl["fwd"] == 4 * t5["d"] * t5["L"] ** 2 * heads
    assert fl["bwd"] == 10 * t5["d"] * t5["L"] ** 2 * heads
