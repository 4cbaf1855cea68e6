"""The narrow tail's host rule and unit decomposition, checked on CPU over
many shapes (the arithmetic the launcher and the kernel's schedule use).

With T tiles and G co-resident clusters, R = T mod G tiles are left for a
last wave.  When 0 < 2 R <= G the launcher asks for T + R units: units
[0, T - R) are whole tiles, and tile T - R + i runs as units T - R + 2 i
(columns [0, BN/2)) and T - R + 2 i + 1 (columns [BN/2, BN)).  Otherwise
units are tiles.  The static schedule hands cluster c the units
c, c + G', c + 2 G', ... with G' = min(units, G); a CLC launch has one
cluster per unit.

* every column of every tile is written by exactly one unit;
* half units appear only when the last wave would leave at least half of the
  clusters idle, and they are the last units handed out;
* on the static schedule no cluster runs more than W whole tiles plus one
  half, so the launch ends about half a tile earlier than with whole tiles.
"""
import pytest


def plan(tiles, resident):
    """(first split tile, parts) as the launcher computes them."""
    rem = tiles % resident
    if rem > 0 and 2 * rem <= resident:
        return tiles - rem, 2
    return tiles, 1


def unit_of(uid, t_first, parts):
    """(tile, half) of unit uid: half -1 is the whole tile."""
    if uid < t_first:
        return uid, -1
    r = uid - t_first
    return t_first + r // parts, r % parts


def num_units(tiles, t_first, parts):
    return t_first + (tiles - t_first) * parts


SHAPES = [1, 2, 30, 37, 38, 73, 74, 75, 90, 100, 111, 112, 147, 148, 150, 180, 222, 256, 296, 300, 304, 400,
          608, 1216]


@pytest.mark.parametrize("tiles", SHAPES)
@pytest.mark.parametrize("resident", [66, 70, 74, 132, 148])
def test_every_column_once(tiles, resident):
    t_first, parts = plan(tiles, resident)
    units = num_units(tiles, t_first, parts)
    seen = {}
    for uid in range(units):
        t, h = unit_of(uid, t_first, parts)
        assert 0 <= t < tiles
        for half in ((0, 1) if h < 0 else (h,)):
            assert (t, half) not in seen, (t, half)
            seen[(t, half)] = uid
    assert len(seen) == 2 * tiles
    # halves only when the last wave is at most half full, and only at the end
    rem = tiles % resident
    assert (parts == 2) == (rem > 0 and 2 * rem <= resident)
    halves = [uid for uid in range(units) if unit_of(uid, t_first, parts)[1] >= 0]
    assert halves == list(range(t_first, units))
    assert len(halves) <= resident


@pytest.mark.parametrize("tiles", SHAPES)
@pytest.mark.parametrize("resident", [66, 74, 148])
def test_static_schedule_ends_half_a_tile_early(tiles, resident):
    t_first, parts = plan(tiles, resident)
    units = num_units(tiles, t_first, parts)
    g = min(units, resident)
    work = [0.0] * g
    for c in range(g):
        for uid in range(c, units, g):
            work[c] += 1.0 if unit_of(uid, t_first, parts)[1] < 0 else 0.5
    assert sum(work) == tiles
    whole_waves = -(-tiles // resident)
    if parts == 2:
        assert max(work) == tiles // resident + 0.5
        assert max(work) == whole_waves - 0.5
    else:
        assert max(work) == whole_waves
