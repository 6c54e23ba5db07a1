"""Pins for the pure-Python tile schedule (hand-computed examples, invariants)."""
import numpy as np

from oracle.schedule import kv_blocks, sample_cost, tile_schedule
from workloads import offsets_from_lengths


def test_hand_example_dense():
    # Lq = 0, 1, 128, 129, 300 with Lk = 64 each; BM = BN = 128, no window.
    ql = [0, 1, 128, 129, 300]
    kl = [64] * 5
    ts, order, cost = tile_schedule(offsets_from_lengths(np.array(ql)),
                                    offsets_from_lengths(np.array(kl)), 128, 128)
    # ntile = 0, 1, 1, 2, 3; each tile sees one key block -> cost 2 per tile.
    assert cost == [0, 2, 2, 4, 6]
    assert order == [4, 3, 1, 2, 0]          # descending cost, ties by sample index
    assert ts == [0, 3, 5, 6, 7, 7]


def test_hand_example_causal_band():
    # One sample of 300 rows = keys, band (127, 0), BM = BN = 128.
    # tile 0 rows 0..127  : keys [0, 128)        -> block 0        -> 1 block
    # tile 1 rows 128..255: keys [1, 256)        -> blocks 0..1    -> 2 blocks
    # tile 2 rows 256..299: keys [129, 300)      -> blocks 1..2    -> 2 blocks
    assert kv_blocks(0, 128, 300, 128, 127, 0) == (0, 1)
    assert kv_blocks(128, 128, 300, 128, 127, 0) == (0, 2)
    assert kv_blocks(256, 128, 300, 128, 127, 0) == (1, 3)
    assert sample_cost(300, 300, 128, 128, 127, 0) == (1 + 1) + (1 + 2) + (1 + 2)


def test_band_beyond_keys_has_no_blocks():
    # right-bounded band, queries far beyond the last key
    assert kv_blocks(256, 128, 10, 64, 0, 0) == (0, 0)
    assert kv_blocks(0, 128, 0, 64, -1, -1) == (0, 0)


def test_order_is_a_permutation_and_prefix_counts_tiles():
    rng = np.random.default_rng(3)
    ql = rng.integers(0, 700, 257)
    kl = rng.integers(0, 900, 257)
    ts, order, cost = tile_schedule(offsets_from_lengths(ql), offsets_from_lengths(kl), 128, 64,
                                    100, 3)
    assert sorted(order) == list(range(257))
    assert all(cost[order[i]] >= cost[order[i + 1]] for i in range(256))
    for i in range(256):
        if cost[order[i]] == cost[order[i + 1]]:
            assert order[i] < order[i + 1]
    ntile = [-(-int(x) // 128) for x in ql]
    assert ts[-1] == sum(ntile)
    assert all(ts[p + 1] - ts[p] == ntile[order[p]] for p in range(257))
