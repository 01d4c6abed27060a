"""The short-segment grouping rule on the CPU: tiles hold whole consecutive segments, never more
than 128 tokens, every short segment lands in exactly one tile, and the greedy cut is maximal."""
import numpy as np
import pytest

from tests import schedule_model as sm


def _check_invariants(lengths):
    cu = np.concatenate([[0], np.cumsum(lengths)])
    us = sm.units(lengths)
    seen = {}
    for u in us:
        if u[0] == "alone":
            assert lengths[u[1]] > 0
            seen[u[1]] = seen.get(u[1], 0) + 1
            continue
        assert len(u[4]) >= 2  # a group shares its tiles between at least two segments
        _, s, n0, ln, segs = u
        assert segs == list(range(s, s + len(segs)))           # consecutive
        assert all(lengths[j] <= sm.TILE for j in segs)         # short only
        assert cu[segs[-1] + 1] - cu[s] == ln                    # contiguous token range
        assert 0 < ln and 0 <= n0 <= sm.TILE and ln - n0 <= sm.TILE
        # the split falls on a segment boundary
        assert any(cu[j] - cu[s] == n0 for j in segs + [segs[-1] + 1])
        for j in segs:
            seen[j] = seen.get(j, 0) + 1
    for i, n in enumerate(lengths):
        if n > 0:
            assert seen.get(i, 0) == 1, (i, n)
    return us


@pytest.mark.parametrize("seed", range(6))
def test_random_packs(seed):
    rng = np.random.default_rng(seed)
    lengths = rng.integers(0, 300, size=400).tolist()
    _check_invariants(lengths)


def test_one_token_segments_fill_tiles():
    us = _check_invariants([1] * 1000)
    # 1000 one-token segments: blocks of 1024 tokens hold them all, so every tile but the
    # last holds 128 tokens (two per group)
    groups = [u for u in us if u[0] == "group"]
    assert [g[3] for g in groups] == [256, 256, 256, 232]
    assert all(g[2] == 128 for g in groups)


def test_greedy_cut_is_maximal():
    lengths = [60, 60, 10, 100, 28, 128, 1]
    us = _check_invariants(lengths)
    # tile 0 = 60 + 60 (the 10 would make 130), tile 1 = 10 + 100; then 28 (128 would make 156),
    # tile 1 = 128; then 1
    assert [(g[2], g[3]) for g in us[:2]] == [(120, 230), (28, 156)]
    assert us[2] == ("alone", 6, 1)  # the last tile holds one segment: it stays alone


def test_long_segments_cut_runs():
    us = _check_invariants([50, 50, 300, 20, 20, 129, 0, 7])
    kinds = [(u[0], u[1]) for u in us]
    # the last run [0, 7] spans two segment indices (one of them empty): a group
    assert kinds == [("group", 0), ("alone", 2), ("group", 3), ("alone", 5), ("group", 6)]
    assert us[-1][3] == 7


def test_block_boundary_cuts_a_run():
    # segments of 100 tokens: starts 0, 100, ..., the one starting at 1100 is the first in
    # block 1 (1024 <= 1100), so a new walk starts there
    lengths = [100] * 15
    us = _check_invariants(lengths)
    starts = [u[1] for u in us]
    assert 11 in starts
    assert sum(u[3] if u[0] == "group" else u[2] for u in us) == 1500
    # the run cut at token 1100 leaves segment 10 (tokens 1000-1099) as the only one of its walk
    assert ("alone", 10, 100) in us


def test_ledger_counts():
    lengths = [0, 5, 0, 130, 0, 0, 257, 0]
    led = sm.ledger(lengths, heads=2)
    # units: [0..3) holds the 5-token segment with two empty ones: a group of several
    # segments; 130 alone, [4..6) empty (no unit), 257 alone, trailing 0: none
    assert led["units"] == 3 and led["groups"] == 1
    assert led["score_tiles"] == 2 * (1 + 4 + 9)
    assert led["items"] == 2 * (1 + 1 + 2)
    assert led["useful_pairs"] == 2 * (25 + 130 ** 2 + 257 ** 2)
    off = sm.ledger(lengths, heads=2, short_packing=False)
    assert off["units"] == 3 and off["groups"] == 0 and off["score_tiles"] == 2 * (1 + 4 + 9)
