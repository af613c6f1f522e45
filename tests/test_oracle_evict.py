"""Pins of the oracle's budget enforcement (CPU only).

Cache What Lasts 2.1 (inference): when the cache exceeds the budget M, the
token with the lowest beta_i^(t-i) is evicted. Pinned by hand-derived cases,
a brute-force minimum of beta^(t-i) evaluated in double as a power (a
different formulation from the float32 log-domain score), FIFO under
constant beta, len = min(M, t+1), and byte checks of the untouched slots.
"""
import json
import os

import numpy as np
import pytest

from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def empty_cache(B, Hkv, cap, d, with_beta=True):
    return dict(k=np.zeros((B, Hkv, cap, d), np.uint16), v=np.zeros((B, Hkv, cap, d), np.uint16),
                log_beta=np.zeros((B, Hkv, cap), np.float32) if with_beta else None,
                pos=np.zeros((B, Hkv, cap), np.int32), len=np.zeros((B, Hkv), np.int32))


def token(seed, t, B, Hkv, d):
    g = rng(seed, t)
    return (normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d)), log_beta(g, (B, Hkv)),
            np.full(B, t, np.int32))


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["evict"], ids=lambda c: c["name"])
def test_closed_forms(oracle, case):
    n = len(case["pos"])
    c = empty_cache(1, 1, n, 8)
    c["pos"][0, 0] = case["pos"]
    c["log_beta"][0, 0] = np.array(case["log_beta"], np.float32)
    c["len"][:] = n
    kn, vn, _, _ = token(0, 0, 1, 1, 8)
    victim = oracle.evict_insert(c, kn, vn, np.array([[-0.5]], np.float32),
                                 np.array([case["t"]], np.int32), M=n)
    assert victim[0, 0] == case["victim"]
    assert c["pos"][0, 0, case["victim"]] == case["t"]


def test_len_is_min_m_t_plus_one(oracle):
    B, Hkv, cap, d, M = 2, 3, 16, 8, 10
    c = empty_cache(B, Hkv, cap, d)
    for t in range(40):
        kn, vn, lb, tt = token(1, t, B, Hkv, d)
        victim = oracle.evict_insert(c, kn, vn, lb, tt, M)
        assert np.all(c["len"] == min(M, t + 1))
        assert np.all((victim == -1) == (t < M))
        for b in range(B):
            for g in range(Hkv):
                p = c["pos"][b, g, :c["len"][b, g]]
                assert len(set(p.tolist())) == len(p) and t in p


def test_victim_has_lowest_retention_bruteforce(oracle):
    B, Hkv, cap, d, M = 2, 2, 32, 4, 32
    c = empty_cache(B, Hkv, cap, d)
    for t in range(M):
        oracle.evict_insert(c, *token(2, t, B, Hkv, d), M)
    for t in range(M, M + 200):
        kn, vn, lb, tt = token(2, t, B, Hkv, d)
        before = {key: c[key].copy() for key in ("k", "v", "log_beta", "pos")}
        victim = oracle.evict_insert(c, kn, vn, lb, tt, M)
        for b in range(B):
            for g in range(Hkv):
                s = victim[b, g]
                beta = np.exp(before["log_beta"][b, g].astype(np.float64))
                ret = np.power(beta, (t - before["pos"][b, g]).astype(np.float64))
                # the victim's retention is the minimum up to float32 rounding of the score
                assert ret[s] <= ret.min() * (1 + 1e-5) + 1e-300
                order = np.argsort(ret)
                if ret[order[1]] > ret[order[0]] * (1 + 1e-4):
                    assert s == order[0]
                # only the victim slot changed, and it now holds the new token
                keep = np.arange(cap) != s
                for key in ("k", "v", "log_beta", "pos"):
                    np.testing.assert_array_equal(c[key][b, g][keep], before[key][b, g][keep])
                np.testing.assert_array_equal(c["k"][b, g, s], kn[b, g])
                np.testing.assert_array_equal(c["v"][b, g, s], vn[b, g])
                assert c["log_beta"][b, g, s] == lb[b, g] and c["pos"][b, g, s] == t


@pytest.mark.parametrize("const", [0.0, -0.3])
def test_constant_beta_is_fifo(oracle, const):
    B, Hkv, cap, d, M = 1, 2, 12, 4, 12
    c = empty_cache(B, Hkv, cap, d)
    for t in range(60):
        kn, vn, _, tt = token(3, t, B, Hkv, d)
        lb = np.full((B, Hkv), const, np.float32)
        oracle.evict_insert(c, kn, vn, lb, tt, M)
        assert sorted(c["pos"][0, 0, :c["len"][0, 0]].tolist()) == list(range(max(0, t + 1 - M), t + 1))


def test_null_log_beta_is_fifo(oracle):
    c = empty_cache(1, 1, 8, 4, with_beta=False)
    for t in range(30):
        kn, vn, _, tt = token(4, t, 1, 1, 4)
        oracle.evict_insert(c, kn, vn, None, tt, 8)
    assert sorted(c["pos"][0, 0].tolist()) == list(range(22, 30))


def test_beta_one_token_survives(oracle):
    c = empty_cache(1, 1, 8, 4)
    for t in range(200):
        kn, vn, lb, tt = token(5, t, 1, 1, 4)
        if t == 3:
            lb[:] = 0.0
        oracle.evict_insert(c, kn, vn, lb, tt, 8)
        if t >= 3:
            assert 3 in c["pos"][0, 0].tolist()


def test_inactive_sequence_untouched(oracle):
    c = empty_cache(2, 1, 4, 4)
    kn, vn, lb, tt = token(6, 0, 2, 1, 4)
    tt[1] = -1
    victim = oracle.evict_insert(c, kn, vn, lb, tt, 4)
    assert c["len"].tolist() == [[1], [0]] and victim.tolist() == [[-1], [-1]]


def test_metadata_only_stream(oracle):
    c = empty_cache(1, 1, 4, 4)
    for t in range(9):
        _, _, lb, tt = token(7, t, 1, 1, 4)
        oracle.evict_insert(c, None, None, lb, tt, 4)
    assert not c["k"].any() and not c["v"].any()
    assert c["len"][0, 0] == 4 and 8 in c["pos"][0, 0].tolist()


def test_invalid_len_is_an_error(oracle):
    c = empty_cache(1, 1, 4, 4)
    c["len"][:] = 5
    with pytest.raises(oracle.OracleError):
        oracle.evict_insert(c, *token(8, 0, 1, 1, 4), 4)
