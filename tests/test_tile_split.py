"""Host-side logic of the token-tile split shared by the increment kernel and
the scan kernel (gla_common.cuh, TileSplit): every tile has one owner, each
CTA's range is contiguous and non-empty, and the partial slot u + c of each
(unit, CTA) pair is unique and below units + CTAs."""

import itertools

import pytest


def lo(c, W, G):
    return (c * W) // G


def owner(x, W, G):
    return ((x + 1) * G - 1) // W


@pytest.mark.parametrize("units,tpu,G", [
    (1008, 29, 148), (840, 13, 148), (5784, 29, 148), (192, 29, 148), (8, 1, 8),
    (2, 1, 2), (7, 3, 5), (1, 1, 1), (3, 40, 148 if 3 * 40 > 148 else 120), (1000, 1, 148),
])
def test_split_properties(units, tpu, G):
    W = units * tpu
    G = min(G, W)
    ranges = [(lo(c, W, G), lo(c + 1, W, G)) for c in range(G)]
    assert ranges[0][0] == 0 and ranges[-1][1] == W
    for (a, b), (c, d) in zip(ranges, ranges[1:]):
        assert b == c
    assert all(b > a for a, b in ranges)  # G <= W: no empty CTA
    slots = set()
    for c, (a, b) in enumerate(ranges):
        for x in range(a, b):
            assert owner(x, W, G) == c
        for u in sorted({x // tpu for x in range(a, b)}):
            s = u + c
            assert s not in slots
            slots.add(s)
            assert s < units + G
    # the scan's view: unit u's partials come from CTAs owner(u*tpu) .. owner(u*tpu + tpu - 1)
    for u in range(units):
        c0, c1 = owner(u * tpu, W, G), owner(u * tpu + tpu - 1, W, G)
        cover = set()
        for c in range(c0, c1 + 1):
            a, b = ranges[c]
            cover |= set(range(max(a, u * tpu), min(b, (u + 1) * tpu)))
        assert cover == set(range(u * tpu, (u + 1) * tpu))


def test_owner_is_inverse_of_lo_exhaustive():
    for W, G in itertools.product(range(1, 60), range(1, 20)):
        if G > W:
            continue
        for x in range(W):
            c = owner(x, W, G)
            assert lo(c, W, G) <= x < lo(c + 1, W, G)
