"""The stream-K schedule's host-side invariants (the arithmetic the kernel
and its launcher use, checked on CPU over many shapes).

The schedule: with G clusters and W = tiles // G >= 2 full waves, the first
(W - 1) G tiles are data-parallel, dealt round robin (cluster c takes c,
c + G, ...); the T = (remaining tiles) x K-block iterations are cut into one
contiguous range [base + c T / G, base + (c + 1) T / G) per cluster.

* the launcher caps the grid at one cluster per 4 iterations (of all the
  tiles), so every cluster's stream-K range is non-empty;
* every (tile, K block) iteration is computed exactly once, by a
  data-parallel tile or a stream-K range;
* a tile's contributors are exactly the consecutive range owners
  owner(first iteration) .. owner(last iteration), which is how the last
  arriver knows how many partials to wait for and sums them in order;
* a split tile is the first or the last stream-K tile of each contributor's
  range, so two partial slots per CTA never collide;
* each cluster runs its split pieces first, then its data-parallel tiles,
  then its whole stream-K tiles.
"""
import pytest


def partition(tiles, nkb, resident):
    G = min(resident, (tiles * nkb + 3) // 4)
    waves = tiles // G
    dp_tiles = (waves - 1) * G if waves >= 2 else 0
    base = dp_tiles * nkb
    T = (tiles - dp_tiles) * nkb
    ranges = [(base + (c * T) // G, base + ((c + 1) * T) // G) for c in range(G)]
    return G, dp_tiles, base, T, ranges


def owner(it, base, T, G):
    return ((it - base + 1) * G + T - 1) // T - 1


SHAPES = [(1, 1), (1, 2), (3, 5), (7, 3), (100, 1), (128, 128), (192, 32), (256, 64), (1000, 7), (148, 16),
          (222, 8), (300, 40)]


@pytest.mark.parametrize("tiles,nkb", SHAPES)
@pytest.mark.parametrize("resident", [70, 74, 148])
def test_stream_k_ranges_contributors_and_slots(tiles, nkb, resident):
    G, dp_tiles, base, T, ranges = partition(tiles, nkb, resident)
    assert dp_tiles % G == 0 and dp_tiles < tiles
    assert all(b > a for a, b in ranges)
    assert ranges[0][0] == base and ranges[-1][1] == base + T == tiles * nkb
    for t in range(dp_tiles, tiles):
        lo, hi = owner(t * nkb, base, T, G), owner((t + 1) * nkb - 1, base, T, G)
        contrib = [c for c, (a, b) in enumerate(ranges) if a < (t + 1) * nkb and b > t * nkb]
        assert contrib == list(range(lo, hi + 1))
        if hi > lo:
            for c in contrib:
                first, last = ranges[c][0] // nkb, (ranges[c][1] - 1) // nkb
                assert t in (first, last)


def run_order(c, G, dp_tiles, ranges, nkb):
    """The order cluster c runs its units: split stream-K pieces (the last,
    then the first), its data-parallel tiles, then its whole stream-K tiles
    in range order -- the sequence the kernel's producer, MMA and epilogue
    roles all walk."""
    lo, hi = ranges[c]
    t0 = lo // nkb
    units = (hi - 1) // nkb - t0 + 1

    def piece(i):
        t = t0 + i
        return t, max(lo - t * nkb, 0), min(hi - t * nkb, nkb)

    whole = lambda p: p[1] == 0 and p[2] == nkb  # noqa: E731
    split_first = units > 0 and not whole(piece(0))
    split_last = units > 1 and not whole(piece(units - 1))
    split = ([units - 1] if split_last else []) + ([0] if split_first else [])
    dp = [(c + k * G, 0, nkb) for k in range(dp_tiles // G)]
    rest = list(range(1 if split_first else 0, units - 1 if split_last else units))
    return [piece(i) for i in split] + dp + [piece(i) for i in rest], len(split)


@pytest.mark.parametrize("tiles,nkb", SHAPES)
@pytest.mark.parametrize("resident", [74, 148])
def test_every_iteration_once_split_pieces_first(tiles, nkb, resident):
    G, dp_tiles, base, T, ranges = partition(tiles, nkb, resident)
    seen = []
    for c in range(G):
        units, n_split = run_order(c, G, dp_tiles, ranges, nkb)
        assert all(not (a == 0 and b == nkb) for _, a, b in units[:n_split])
        assert all(a == 0 and b == nkb for _, a, b in units[n_split:])
        seen += [(t, k) for t, a, b in units for k in range(a, b)]
    assert sorted(seen) == [(t, k) for t in range(tiles) for k in range(nkb)]
