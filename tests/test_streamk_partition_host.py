"""The stream-K schedule's host-side invariants (the arithmetic the kernel
and its launcher use, checked on CPU over many shapes):

* the launcher caps the grid at one cluster per 4 iterations, so every
  cluster's range [c T / G, (c + 1) T / G) of the T = tiles x K-block
  iterations is non-empty;
* a tile's contributors are exactly the consecutive range owners
  owner(first iteration) .. owner(last iteration), which is how the last
  arriver knows how many partials to wait for and sums them in order;
* a split tile is the first or the last tile of each contributor's range,
  so two partial slots per CTA never collide.
"""
import pytest


def partition(tiles, nkb, resident):
    T = tiles * nkb
    G = min(resident, (T + 3) // 4)
    return T, G, [((c * T) // G, ((c + 1) * T) // G) for c in range(G)]


def owner(it, T, G):
    return ((it + 1) * G + T - 1) // T - 1


@pytest.mark.parametrize("tiles,nkb", [(1, 1), (1, 2), (3, 5), (7, 3), (100, 1), (128, 128), (192, 32),
                                       (256, 64), (1000, 7)])
@pytest.mark.parametrize("resident", [70, 74, 148])
def test_stream_k_ranges_contributors_and_slots(tiles, nkb, resident):
    T, G, ranges = partition(tiles, nkb, resident)
    assert all(b > a for a, b in ranges)
    assert ranges[0][0] == 0 and ranges[-1][1] == T
    for t in range(tiles):
        lo, hi = owner(t * nkb, T, G), owner((t + 1) * nkb - 1, T, G)
        contrib = [c for c, (a, b) in enumerate(ranges) if a < (t + 1) * nkb and b > t * nkb]
        assert contrib == list(range(lo, hi + 1))
        if hi > lo:
            for c in contrib:
                first, last = ranges[c][0] // nkb, (ranges[c][1] - 1) // nkb
                assert t in (first, last)


def run_order(lo, hi, nkb):
    """The order a cluster runs the pieces of its range [lo, hi): split
    pieces (the last, then the first) before the whole tiles, the rest in
    range order -- the sequence the kernel's producer, MMA and epilogue
    roles all walk."""
    t0 = lo // nkb
    units = (hi - 1) // nkb - t0 + 1

    def piece(i):
        t = t0 + i
        return t, max(lo - t * nkb, 0), min(hi - t * nkb, nkb)

    whole = lambda p: p[1] == 0 and p[2] == nkb  # noqa: E731
    split_first = units > 0 and not whole(piece(0))
    split_last = units > 1 and not whole(piece(units - 1))
    order = ([units - 1] if split_last else []) + ([0] if split_first else [])
    order += list(range(1 if split_first else 0, units - 1 if split_last else units))
    return [piece(i) for i in order], split_first, split_last


@pytest.mark.parametrize("tiles,nkb", [(1, 2), (3, 5), (7, 3), (128, 128), (192, 32), (256, 64)])
def test_stream_k_runs_each_piece_once_split_pieces_first(tiles, nkb):
    T, G, ranges = partition(tiles, nkb, 74)
    for lo, hi in ranges:
        pieces, split_first, split_last = run_order(lo, hi, nkb)
        covered = sorted((t * nkb + a, t * nkb + b) for t, a, b in pieces)
        assert covered[0][0] == lo and covered[-1][1] == hi
        assert all(x[1] == y[0] for x, y in zip(covered, covered[1:]))      # each iteration once
        n_split = int(split_first) + int(split_last)
        assert all(not (a == 0 and b == nkb) for _, a, b in pieces[:n_split])
        assert all(a == 0 and b == nkb for _, a, b in pieces[n_split:])
