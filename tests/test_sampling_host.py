"""The token sampling of the large-batch parity tests: every (expert, 128-row M tile) of the
permuted order gets a checked row, and at least 512 tokens are checked."""
import numpy as np

from helpers import expert_segments, tile_covering_tokens, uncovered_tiles


def skewed_ids(T, rng):
    # two hot experts (3 and 11) take most assignments, as in the skewed-routing workload
    p = np.full(16, 1.0)
    p[[3, 11]] = 14.0
    p /= p.sum()
    ids = np.empty((T, 2), np.int32)
    for t in range(T):
        ids[t] = rng.choice(16, 2, replace=False, p=p)
    return ids


def test_segments_are_stable_token_order():
    ids = np.array([[3, 1], [1, 3], [0, 3]], np.int32)
    seg = expert_segments(ids)
    assert seg[3].tolist() == [0, 3, 5] and seg[1].tolist() == [1, 2] and seg[0].tolist() == [4]


def test_every_tile_covered_and_at_least_512():
    rng = np.random.default_rng(1)
    ids = skewed_ids(20000, rng)
    toks = tile_covering_tokens(ids)
    assert toks.size >= 512 and np.unique(toks).size == toks.size
    assert uncovered_tiles(ids, toks) == []
    n_tiles = sum((s.size + 127) // 128 for s in expert_segments(ids))
    assert toks.size >= n_tiles // 2  # a token covers at most one tile of each of its two experts


def test_uncovered_tiles_detects_a_gap():
    rng = np.random.default_rng(2)
    ids = skewed_ids(3000, rng)
    toks = tile_covering_tokens(ids, n_min=0)
    seg3 = expert_segments(ids)[3]
    tile1 = set((seg3[128:256] // 2).tolist())
    kept = np.array([t for t in toks if t not in tile1])
    assert (3, 1) in uncovered_tiles(ids, kept)


def test_small_batch_takes_every_token():
    ids = np.stack([np.arange(40) % 16, (np.arange(40) + 1) % 16], 1).astype(np.int32)
    assert tile_covering_tokens(ids).tolist() == list(range(40))


def test_dense_mlp_single_expert():
    ids = np.zeros((8192, 1), np.int32)
    toks = tile_covering_tokens(ids)
    assert toks.size >= 512 and uncovered_tiles(ids, toks) == []
