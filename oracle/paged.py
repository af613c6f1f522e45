"""Oracle view of a paged cache (MEMENTO, systems section: KV entries removed inside generation;
the cache is a sawtooth): the logical cache of each (sequence b, kv head g) -- slots [0, len) in
slot order -- is kept in pages of PAGE slots drawn from one pool, logical slot s being row s % PAGE
of page table[b, g, s // PAGE]. Every paged operation is defined as its flat counterpart on the
logical cache, so the oracle of the paged path is the flat oracle (kvb_oracle.cpp) applied to this
view; this module only maps between the two layouts.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py). Plain numpy, no arithmetic of the method.
"""
from __future__ import annotations

import numpy as np

PAGE = 64


def to_flat(pages: dict, table, len_, cap: int | None = None) -> dict:
    """The logical (flat) cache of a paged one.

    pages: {"k", "v": [P, PAGE, d] uint16; "pos": [P, PAGE] int32; "log_beta": [P, PAGE] float32 or
    None}; table [B, Hkv, max_pages] int; len [B, Hkv]. Returns {"k", "v" [B, Hkv, cap, d], "pos",
    "log_beta" [B, Hkv, cap], "len"} with slots at or beyond len zero (cap defaults to max_pages *
    PAGE). Raises ValueError when a slot below len lies in a page the table does not name."""
    table = np.asarray(table)
    len_ = np.asarray(len_)
    B, Hkv, max_pages = table.shape
    cap = max_pages * PAGE if cap is None else cap
    d = pages["k"].shape[-1]
    out = dict(k=np.zeros((B, Hkv, cap, d), np.uint16), v=np.zeros((B, Hkv, cap, d), np.uint16),
               pos=np.zeros((B, Hkv, cap), np.int32),
               log_beta=None if pages.get("log_beta") is None else np.zeros((B, Hkv, cap), np.float32),
               len=len_.astype(np.int32).copy())
    P = pages["k"].shape[0]
    for b in range(B):
        for g in range(Hkv):
            n = int(len_[b, g])
            for s in range(n):
                pg = int(table[b, g, s // PAGE])
                if not 0 <= pg < P:
                    raise ValueError(f"slot {s} of (b={b}, g={g}) is in no page of the pool")
                r = s % PAGE
                out["k"][b, g, s] = pages["k"][pg, r]
                out["v"][b, g, s] = pages["v"][pg, r]
                out["pos"][b, g, s] = pages["pos"][pg, r]
                if out["log_beta"] is not None:
                    out["log_beta"][b, g, s] = pages["log_beta"][pg, r]
    return out


def from_flat(flat: dict, page_order, num_pages: int) -> tuple[dict, np.ndarray]:
    """A paged copy of a flat cache: the logical pages of (b, g) in row-major order take the pool
    pages page_order[0], page_order[1], ... Returns (pages, table)."""
    B, Hkv, cap, d = flat["k"].shape
    max_pages = -(-cap // PAGE)
    pages = dict(k=np.zeros((num_pages, PAGE, d), np.uint16), v=np.zeros((num_pages, PAGE, d), np.uint16),
                 pos=np.zeros((num_pages, PAGE), np.int32),
                 log_beta=None if flat.get("log_beta") is None else np.zeros((num_pages, PAGE), np.float32))
    table = np.full((B, Hkv, max_pages), -1, np.int32)
    it = iter(page_order)
    for b in range(B):
        for g in range(Hkv):
            n = int(flat["len"][b, g])
            for j in range(-(-n // PAGE)):
                pg = int(next(it))
                table[b, g, j] = pg
                rows = slice(j * PAGE, min(n, (j + 1) * PAGE))
                m = rows.stop - rows.start
                pages["k"][pg, :m] = flat["k"][b, g, rows]
                pages["v"][pg, :m] = flat["v"][b, g, rows]
                pages["pos"][pg, :m] = flat["pos"][b, g, rows]
                if pages["log_beta"] is not None:
                    pages["log_beta"][pg, :m] = flat["log_beta"][b, g, rows]
    return pages, table
