"""Host-side checks of the stream-K work split that the small-M, tile and pair
kernels share (no GPU needed).

U = T x nkb (tile, k-block) units are dealt to G CTAs (pairs) as contiguous
ranges [g U / G, (g + 1) U / G). The kernels find the CTA that holds unit u
with the closed form owner(u) = ((u + 1) G - 1) / U (integer division; the
device evaluates it in double precision), and a tile's partial-sum slot of
CTA g is g - owner(first unit of the tile). These tests check, on the launch
shapes the library uses and on random ones, that the closed form agrees with
the ranges, that the double-precision form is exact, and that the segments of
every tile are numbered 0 .. nseg - 1 with each unit held by exactly one CTA.
"""
import random

import pytest


def owner_int(u, G, U):
    return ((u + 1) * G - 1) // U


def owner_double(u, G, U):
    return int((float(u + 1) * G - 1.0) / float(U))


def ranges(G, U):
    return [(g * U // G, (g + 1) * U // G) for g in range(G)]


def segments(G, T, nkb):
    """Per CTA, its (tile, kb0, nk, slot, nseg) segments, as the kernels walk them."""
    U = T * nkb
    out = []
    for g, (u, u1) in enumerate(ranges(G, U)):
        segs = []
        while u < u1:
            t = u // nkb
            end = min((t + 1) * nkb, u1)
            first = owner_int(t * nkb, G, U)
            last = owner_int((t + 1) * nkb - 1, G, U)
            segs.append((t, u - t * nkb, end - u, g - first, last - first + 1))
            u = end
        out.append(segs)
    return out


# (G, T, nkb): 74 pairs over the 70B QKV tiles at M = 256 (20 tiles x 256 k-blocks of 32) and the 12
# left over at M = 2048; 148 CTAs over the 8B decode's 48 W tiles x 64 k-blocks; odd and tiny cases
SHAPES = [(74, 20, 256), (74, 12, 256), (74, 32, 128), (74, 2, 64), (148, 48, 64), (148, 80, 128),
          (148, 3, 64), (7, 5, 3), (3, 1, 3), (5, 4, 1)]


@pytest.mark.parametrize("G,T,nkb", SHAPES)
def test_owner_matches_the_ranges(G, T, nkb):
    U = T * nkb
    if U < G:
        pytest.skip("fewer units than CTAs: the kernels reject this split")
    for g, (u0, u1) in enumerate(ranges(G, U)):
        assert u1 > u0
        for u in range(u0, u1):
            assert owner_int(u, G, U) == g
            assert owner_double(u, G, U) == g


@pytest.mark.parametrize("G,T,nkb", SHAPES)
def test_segments_cover_each_unit_once_with_contiguous_slots(G, T, nkb):
    U = T * nkb
    if U < G:
        pytest.skip("fewer units than CTAs")
    held = [[None] * nkb for _ in range(T)]
    slots = {}
    for g, segs in enumerate(segments(G, T, nkb)):
        for t, kb0, nk, slot, nseg in segs:
            for kb in range(kb0, kb0 + nk):
                assert held[t][kb] is None
                held[t][kb] = g
            slots.setdefault(t, []).append((slot, nseg, g))
    assert all(h is not None for row in held for h in row)
    for t, lst in slots.items():
        nseg = lst[0][1]
        assert all(n == nseg for _, n, _ in lst)
        assert sorted(s for s, _, _ in lst) == list(range(nseg))
        # slot order is CTA order, so a tile's slots are summed in k order
        assert [g for _, _, g in sorted(lst)] == sorted(g for _, _, g in lst)


def test_double_owner_is_exact_on_large_random_splits():
    rng = random.Random(7)
    for _ in range(20000):
        G = rng.randint(1, 4096)
        U = rng.randint(G, 1 << 40)
        u = rng.randrange(U)
        assert owner_double(u, G, U) == owner_int(u, G, U), (u, G, U)
    for G, U in ((74, 5120), (148, 3072), (148, 1 << 30)):   # range edges
        for g in range(G):
            for u in (g * U // G, (g + 1) * U // G - 1):
                assert owner_double(u, G, U) == owner_int(u, G, U) == g
