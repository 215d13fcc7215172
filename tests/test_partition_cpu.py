"""The split-N partition of the state reduction, re-derived independently:
CTA c of G owns items [floor(c*I/G), floor((c+1)*I/G)); its partial for head
bh goes to slot c + bh; the combine of head bh reads CTAs cta_of(first item)
.. cta_of(last item).  Checks that every item is reduced exactly once, slots
never collide, and the combine ranges hold exactly the CTAs that wrote a
partial for the head."""
import random

import pytest


def segments(BH, tph, G):
    items = BH * tph
    segs = []
    for c in range(G):
        lo, hi = c * items // G, (c + 1) * items // G
        w = lo
        while w < hi:
            bh = w // tph
            end = min(hi, (bh + 1) * tph)
            segs.append((c, bh, w, end))
            w = end
    return segs


def cta_of(w, G, items):
    return ((w + 1) * G - 1) // items


@pytest.mark.parametrize("seed", range(40))
def test_partition_invariants(seed):
    rnd = random.Random(seed)
    BH = rnd.randint(1, 64)
    tph = rnd.randint(1, 500)
    items = BH * tph
    G = rnd.randint(1, min(items, 512))
    segs = segments(BH, tph, G)
    covered = [0] * items
    for c, bh, lo, hi in segs:
        for w in range(lo, hi):
            covered[w] += 1
    assert all(x == 1 for x in covered)
    slots = [c + bh for c, bh, _, _ in segs]
    assert len(set(slots)) == len(slots)
    assert max(slots) < G + BH
    for bh in range(BH):
        writers = sorted(c for c, b, _, _ in segs if b == bh)
        lo = cta_of(bh * tph, G, items)
        hi = cta_of((bh + 1) * tph - 1, G, items)
        assert writers == list(range(lo, hi + 1))


def test_cta_of_matches_ranges():
    for items in (1, 7, 148, 4600, 14043):
        for G in sorted({1, min(items, 3), min(items, 148), min(items, 512)}):
            for w in range(items):
                c = cta_of(w, G, items)
                assert c * items // G <= w < (c + 1) * items // G
