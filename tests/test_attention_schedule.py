"""Host-side check of the prefill attention kernel's item schedule (no GPU).

Work items are (query tile, batch row, head), heaviest causal query tiles
first.  CTA c of G takes one item per round of G in snake order: round i
gives it item i*G + c, or i*G + G - 1 - c when i is odd.  Its item count is
the number of full rounds plus one when the partial last round reaches it.
Restated here from that definition: every item is taken exactly once, and
on the 7B prefill shape the longest CTA walks 31 key tiles (38 with a plain
stride), the figure the kernel's documentation quotes.
"""
import pytest


def _items(NW, G, c):
    full, rem = NW // G, NW % G
    last = rem > 0 and ((G - 1 - c) < rem if full & 1 else c < rem)
    n = full + (1 if last else 0)
    return [i * G + (G - 1 - c if i & 1 else c) for i in range(n)]


def _key_tiles(k, qtiles, BH, causal=True):
    qt = qtiles - 1 - k // BH
    return qt + 1 if causal else qtiles


@pytest.mark.parametrize("NW,G", [(1, 1), (7, 7), (148, 148), (149, 148), (295, 148), (296, 148),
                                  (512, 148), (1536, 148), (2048, 132), (97, 64), (6144, 148)])
def test_every_item_once(NW, G):
    seen = []
    for c in range(G):
        ks = _items(NW, G, c)
        assert all(0 <= k < NW for k in ks)
        seen += ks
    assert sorted(seen) == list(range(NW))


def test_snake_balances_causal_7b_prefill():
    # 2048 tokens: 16 query tiles of 128, 32 heads, B = 1, 148 SMs
    qtiles, BH, G = 16, 32, 148
    NW = qtiles * BH
    snake = [sum(_key_tiles(k, qtiles, BH) for k in _items(NW, G, c)) for c in range(G)]
    stride = [sum(_key_tiles(k, qtiles, BH) for k in range(c, NW, G)) for c in range(G)]
    assert sum(snake) == sum(stride) == BH * qtiles * (qtiles + 1) // 2
    assert max(snake) == 31 and max(stride) == 38


def test_grid_smaller_than_items_count():
    # fewer items than SMs: the grid is the item count, one item per CTA
    for NW in (1, 5, 100):
        assert [len(_items(NW, NW, c)) for c in range(NW)] == [1] * NW
