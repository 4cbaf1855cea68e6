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
