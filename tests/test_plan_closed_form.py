"""The split-KV work plan's closed forms (csrc/split_plan.cuh) against their definition by
search, on the host: a sequence's first unit is the last unit whose first tile is at or
before the sequence's first tile, its slot count the units from there to the unit holding its
last tile, and a unit's first sequence the last sequence starting at or before the unit's
first tile. Balanced plans cut the tile space into units of `per` tiles; capped plans cut each
sequence alone into min(max_splits, tiles) near-equal ranges. Random ragged batches, empty
sequences included."""

import numpy as np
import pytest

TILE = 64


def _upper_index(v, t):
    """Largest i with v[i] <= t (v non-decreasing, v[0] <= t)."""
    i = 0
    for j, x in enumerate(v):
        if x <= t:
            i = j
    return i


def _cut(lens, units_target, max_splits):
    tiles = [(L + TILE - 1) // TILE for L in lens]
    tstart = np.concatenate([[0], np.cumsum(tiles)]).astype(int)
    total = int(tstart[-1])
    if total == 0:
        return tiles, tstart, [total], 0
    if max_splits == 0:
        per = (total + units_target - 1) // units_target
        n_units = (total + per - 1) // per
        begin = [u * per for u in range(n_units)]
    else:
        begin, per = [], 0
        for b, t in enumerate(tiles):
            n = min(t, max_splits)
            begin += [int(tstart[b]) + (k * t) // n for k in range(n)]
    return tiles, tstart, begin + [total], per


def _by_search(lens, units_target, max_splits):
    tiles, tstart, begin, _ = _cut(lens, units_target, max_splits)
    n_units = len(begin) - 1
    first, slots = [], []
    for b, t in enumerate(tiles):
        if t == 0:
            first.append(0)
            slots.append(0)
            continue
        f = _upper_index(begin[:n_units], int(tstart[b]))
        last = _upper_index(begin[:n_units], int(tstart[b]) + t - 1)
        first.append(f)
        slots.append(last - f + 1)
    unit_seq = [_upper_index(tstart[:len(lens)], begin[u]) for u in range(n_units)]
    return first, slots, unit_seq


def _closed_form(lens, units_target, max_splits):
    tiles, tstart, begin, per = _cut(lens, units_target, max_splits)
    n_units = len(begin) - 1
    first, slots, unit_seq = [], [], [0] * n_units
    capped_start = np.concatenate([[0], np.cumsum([min(t, max_splits) for t in tiles])]).astype(int)
    for b, t in enumerate(tiles):
        if t == 0:
            first.append(0)
            slots.append(0)
        elif max_splits == 0:
            f = int(tstart[b]) // per
            first.append(f)
            slots.append((int(tstart[b]) + t - 1) // per - f + 1)
        else:
            first.append(int(capped_start[b]))
            slots.append(min(t, max_splits))
        if max_splits > 0:
            for k in range(min(t, max_splits)):
                unit_seq[int(capped_start[b]) + k] = b
    if max_splits == 0:
        unit_seq = [_upper_index(tstart[:len(lens)], u * per) for u in range(n_units)]
    return first, slots, unit_seq


@pytest.mark.parametrize("max_splits", [0, 1, 3, 16])
def test_closed_forms_equal_the_search(max_splits):
    rng = np.random.default_rng(5 + max_splits)
    for _ in range(200):
        batch = int(rng.integers(1, 40))
        lens = [int(x) if rng.random() > 0.15 else 0 for x in rng.integers(1, 3000, batch)]
        units = int(rng.integers(1, 80))
        assert _closed_form(lens, units, max_splits) == _by_search(lens, units, max_splits), (lens, units)


def test_a_planted_off_by_one_is_caught():
    """The last tile of a sequence taken as tstart + tiles (one past it): the slot counts then
    disagree with the search on some batch, so the comparison above has teeth."""
    rng = np.random.default_rng(11)
    caught = False
    for _ in range(200):
        batch = int(rng.integers(1, 40))
        lens = [int(x) for x in rng.integers(1, 3000, batch)]
        units = int(rng.integers(2, 80))
        tiles, tstart, _, per = _cut(lens, units, 0)
        wrong = [(int(tstart[b]) + t) // per - int(tstart[b]) // per + 1 for b, t in enumerate(tiles)]
        if wrong != _by_search(lens, units, 0)[1]:
            caught = True
            break
    assert caught
