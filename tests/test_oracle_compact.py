"""Pins of the oracle's in-place block removal (CPU only).

MEMENTO (chunking and compression; dual information stream): a finished
block's KV entries are physically removed in place and the memento entries
after it are kept bit for bit. Pinned against numpy.delete on the slot axis,
and by attention after compaction == SDPA over the old cache with the removed
keys masked out.
"""
import math

import numpy as np
import pytest

from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from refs import f64, sdpa_state


def random_cache(seed, B, Hkv, cap, d, n):
    g = rng(seed, 5)
    return dict(k=normal_bf16(g, (B, Hkv, cap, d)), v=normal_bf16(g, (B, Hkv, cap, d)),
                log_beta=log_beta(g, (B, Hkv, cap)),
                pos=np.tile(np.arange(cap, dtype=np.int32), (B, Hkv, 1)),
                len=np.full((B, Hkv), n, np.int32))


@pytest.mark.parametrize("r0,rl", [(0, 0), (3, 5), (0, 40), (10, 2), (30, 10), (1, 1), (0, 1), (38, 2)])
def test_matches_numpy_delete(oracle, r0, rl):
    B, Hkv, cap, d, n = 3, 2, 48, 8, 40
    c = random_cache(1, B, Hkv, cap, d, n)
    before = {key: val.copy() for key, val in c.items()}
    rs = np.array([r0, 0, r0], np.int32)
    rls = np.array([rl, 0, rl], np.int32)
    oracle.compact_blocks(c, rs, rls)
    for b in range(B):
        for g in range(Hkv):
            rem = np.arange(rs[b], rs[b] + rls[b])
            m = n - rls[b]
            assert c["len"][b, g] == m
            for key in ("k", "v", "log_beta", "pos"):
                exp = np.delete(before[key][b, g, :n], rem, axis=0)
                np.testing.assert_array_equal(c[key][b, g, :m], exp)
                # slots beyond the new length are not read; slots beyond the old length are untouched
                np.testing.assert_array_equal(c[key][b, g, n:], before[key][b, g, n:])


@pytest.mark.parametrize("r0,rl", [(-1, 2), (5, 36), (41, 0 + 1), (0, -3)])
def test_invalid_range_is_an_error_and_a_no_op(oracle, r0, rl):
    c = random_cache(2, 1, 2, 48, 8, 40)
    before = {key: val.copy() for key, val in c.items()}
    with pytest.raises(oracle.OracleError):
        oracle.compact_blocks(c, np.array([r0], np.int32), np.array([rl], np.int32))
    for key in before:
        np.testing.assert_array_equal(c[key], before[key])


def test_attention_after_compaction_equals_masked_attention(oracle):
    B, Hkv, cap, d, n = 1, 2, 64, 32, 60
    c = random_cache(3, B, Hkv, cap, d, n)
    old = {key: val.copy() for key, val in c.items()}
    q = normal_bf16(rng(3, 6), (B, 8, d))
    oracle.compact_blocks(c, np.array([12], np.int32), np.array([30], np.int32))
    o, lse = oracle.decode_attn(q, c["k"], c["v"], None, c["pos"], c["len"], None)
    keep = np.r_[0:12, 42:60]
    for h in range(8):
        g = h // 4
        eo, el = sdpa_state(f64(q[0, h])[None], f64(old["k"][0, g, keep]), f64(old["v"][0, g, keep]),
                            1 / math.sqrt(d))
        np.testing.assert_allclose(o[0, h], eo[0], atol=1e-12)
        np.testing.assert_allclose(lse[0, h], el[0], atol=1e-12)
