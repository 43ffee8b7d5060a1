"""Host-side invariants of the stream-K work split (no GPU).

The stream-K plan gives CTA j of G the run of global tiles
[j W / G, (j + 1) W / G) of the W = rows x nt tiles laid end to end, finds
the CTA that owns global tile g as ((g + 1) G - 1) / W, keeps a shared row's
parts in slots 2 j (the row is CTA j's first) or 2 j + 1 (its last), and is
offered only when rows > G / 2, so that a row falls to at most three CTAs
(the kernel merges at most three parts).  These checks restate those integer
formulas and confirm, over many shapes, that ownership is a partition, that
the part count stays within three, and that the slot a part is written to is
the slot the merging CTA reads."""
import itertools

import pytest

MAX_PIECES = 3


def start(j, W, G):
    return j * W // G


def owner(g, W, G):
    return ((g + 1) * G - 1) // W


def streamk_offered(rows, nt, G):
    return nt >= 16 and 2 * rows > G and rows % G != 0 and rows * nt < (1 << 31)


def writer_slot(j, r, W, G, nt):
    b0 = start(j, W, G) // nt            # the CTA's first row
    return 2 * j + (0 if r == b0 else 1)


def reader_slot(j, r, W, G, nt):
    return 2 * j + (0 if start(j, W, G) // nt == r else 1)


SHAPES = [(rows, nt, G) for G in (148, 132, 7) for nt in (16, 17, 32, 40)
          for rows in sorted({G // 2 + 1, G // 2 + 13, G - 20, G - 1, G + 1, G + 2, 2 * G - 3, 3 * G + 5})]


@pytest.mark.parametrize("rows,nt,G", SHAPES)
def test_ownership_partitions_the_tiles(rows, nt, G):
    if not streamk_offered(rows, nt, G):
        pytest.skip("plan not offered")
    W = rows * nt
    counts = [start(j + 1, W, G) - start(j, W, G) for j in range(G)]
    assert sum(counts) == W and min(counts) >= 1 and max(counts) - min(counts) <= 1
    for j in range(G):
        for g in (start(j, W, G), start(j + 1, W, G) - 1):
            assert owner(g, W, G) == j


@pytest.mark.parametrize("rows,nt,G", SHAPES)
def test_pieces_and_slots(rows, nt, G):
    if not streamk_offered(rows, nt, G):
        pytest.skip("plan not offered")
    W = rows * nt
    used = {}
    for r in range(rows):
        j0, j1 = owner(r * nt, W, G), owner((r + 1) * nt - 1, W, G)
        assert 1 <= j1 - j0 + 1 <= MAX_PIECES, (r, j0, j1)
        if j0 == j1:
            continue                                  # written out directly, no slot
        for j in range(j0, j1 + 1):
            # the CTA's tiles of row r form one run, at the start or the end of its range
            lo, hi = max(start(j, W, G), r * nt), min(start(j + 1, W, G), (r + 1) * nt)
            assert lo < hi
            assert lo == start(j, W, G) or hi == start(j + 1, W, G)
            s = writer_slot(j, r, W, G, nt)
            assert s == reader_slot(j, r, W, G, nt)
            assert 0 <= s < 2 * G
            assert s not in used, (s, used.get(s), (r, j))
            used[s] = (r, j)


def test_offer_rule_examples():
    assert streamk_offered(128, 32, 148)              # c5: 20 idle SMs
    assert not streamk_offered(148, 32, 148)          # one full wave already
    assert not streamk_offered(74, 32, 148)           # the cluster split plan
    assert not streamk_offered(128, 15, 148)          # lists shorter than 16 tiles
    # more than three parts would need rows <= G / 2, which is never offered
    for rows, nt in itertools.product(range(75, 300, 7), (16, 24, 32)):
        if streamk_offered(rows, nt, 148):
            W = rows * nt
            assert max(owner((r + 1) * nt - 1, W, 148) - owner(r * nt, W, 148) for r in range(rows)) < MAX_PIECES
