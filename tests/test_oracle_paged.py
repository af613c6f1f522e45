"""Pins of the oracle's paged view (oracle/paged.py): the logical cache of a paged cache.
A hand-built table whose answer is written out slot by slot, a round trip through a random
page order, and the view of a cache whose pages are out of order and partly used."""
import numpy as np
import pytest

from oracle import paged


def test_hand_built_table_maps_slots_to_page_rows():
    # one (b, g) with 130 slots in pages 2, 0, 1 (in that order): slot s -> page [2, 0, 1][s // 64], row s % 64
    P, d = 3, 8
    k = np.zeros((P, 64, d), np.uint16)
    pos = np.zeros((P, 64), np.int32)
    for pg in range(P):
        for r in range(64):
            k[pg, r] = 1000 * pg + r
            pos[pg, r] = 100 * pg + r
    pages = dict(k=k, v=k + 7, pos=pos, log_beta=None)
    flat = paged.to_flat(pages, np.array([[[2, 0, 1]]]), np.array([[130]]))
    assert flat["k"][0, 0, 0, 0] == 2000 and flat["k"][0, 0, 63, 0] == 2063   # page 2, rows 0 and 63
    assert flat["k"][0, 0, 64, 0] == 0 and flat["k"][0, 0, 127, 0] == 63      # page 0
    assert flat["k"][0, 0, 128, 0] == 1000 and flat["k"][0, 0, 129, 0] == 1001  # page 1, partly used
    assert flat["pos"][0, 0, 129] == 101 and flat["v"][0, 0, 5, 3] == 2012
    assert not flat["k"][0, 0, 130:].any() and flat["len"][0, 0] == 130


def test_round_trip_through_a_random_page_order():
    g = np.random.default_rng(0)
    B, Hkv, cap, d = 3, 2, 256, 16
    n = np.array([[256, 0], [65, 64], [1, 130]], np.int32)
    flat = dict(k=g.integers(0, 2 ** 16, (B, Hkv, cap, d), dtype=np.uint16),
                v=g.integers(0, 2 ** 16, (B, Hkv, cap, d), dtype=np.uint16),
                pos=g.integers(0, 10 ** 6, (B, Hkv, cap), dtype=np.int32),
                log_beta=g.standard_normal((B, Hkv, cap)).astype(np.float32), len=n)
    for key in ("k", "v", "pos", "log_beta"):   # slots beyond len are not part of the cache
        for b in range(B):
            for h in range(Hkv):
                flat[key][b, h, n[b, h]:] = 0
    need = int(sum(-(-x // 64) for x in n.ravel()))
    order = g.permutation(need + 5)[:need]
    pages, table = paged.from_flat(flat, order, need + 5)
    back = paged.to_flat(pages, table, n, cap)
    for key in ("k", "v", "pos", "log_beta", "len"):
        np.testing.assert_array_equal(back[key], flat[key], err_msg=key)
    # every page used at most once, and exactly the pages the lengths need
    used = table[table >= 0]
    assert len(np.unique(used)) == used.size == need


def test_a_slot_outside_the_pool_is_an_error():
    pages = dict(k=np.zeros((1, 64, 8), np.uint16), v=np.zeros((1, 64, 8), np.uint16),
                 pos=np.zeros((1, 64), np.int32), log_beta=None)
    with pytest.raises(ValueError):
        paged.to_flat(pages, np.array([[[0, -1]]]), np.array([[65]]))
