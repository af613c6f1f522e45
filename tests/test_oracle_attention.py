"""Pins of the oracle's decode attention (CPU only).

The oracle is checked against things other than itself: hand-derived closed
forms (tests/golden/closed_forms.json), torch's scaled_dot_product_attention in
float64 (plain and with the retention bias as an additive mask), the
online-softmax identity (merging per-split states reproduces the unsplit
state), and structural invariants (GQA isolation, empty and inactive rows,
a shared cache through batch stride 0).
"""
import json
import math
import os

import numpy as np
import pytest

from memory_bounded_kv_b200.synth import to_bf16_bits, normal_bf16, log_beta, rng
from refs import f64, sdpa_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _ev(x):
    if x is None:
        return None
    return float(eval(str(x), {"__builtins__": {}}, {**vars(math), "inf": math.inf}))


def _random_cache(seed, B, Hq, Hkv, d, cap, lens, with_beta=True):
    g = rng(seed, 99)
    q = normal_bf16(g, (B, Hq, d))
    k = normal_bf16(g, (B, Hkv, cap, d))
    v = normal_bf16(g, (B, Hkv, cap, d))
    lb = log_beta(g, (B, Hkv, cap)) if with_beta else None
    t = np.full(B, 3 * cap, np.int32)
    pos = np.stack([np.stack([g.permutation(3 * cap)[:cap] for _ in range(Hkv)]) for _ in range(B)]).astype(np.int32)
    ln = np.asarray(lens, np.int32).reshape(B, Hkv)
    return q, k, v, lb, pos, ln, t


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["attention"], ids=lambda c: c["name"])
def test_closed_forms(oracle, case):
    q = to_bf16_bits(np.array(case["q"], np.float32))[None]            # [1, Hq, d]
    k = to_bf16_bits(np.array(case["k"], np.float32))[None, None]      # [1, 1, n, d]
    v = to_bf16_bits(np.array(case["v"], np.float32))[None, None]
    n = k.shape[2]
    lb = None if case["log_beta"] is None else np.array([_ev(x) for x in case["log_beta"]], np.float32)[None, None]
    pos = np.array(case["pos"], np.int32)[None, None]
    o, lse = oracle.decode_attn(q, k, v, lb, pos, np.array([[n]], np.int32), np.array([case["t"]], np.int32),
                                scale=case["scale"])
    exp_o = np.array([[_ev(x) for x in row] for row in case["o"]])
    exp_l = np.array([_ev(x) for x in case["lse"]])
    np.testing.assert_allclose(o[0], exp_o, rtol=0, atol=1e-7)
    np.testing.assert_allclose(lse[0], exp_l, rtol=0, atol=1e-7)


@pytest.mark.parametrize("d", [4, 16, 64, 128])
@pytest.mark.parametrize("with_beta", [False, True])
def test_matches_sdpa(oracle, d, with_beta):
    B, Hq, Hkv, cap = 2, 8, 2, 40
    lens = [[40, 1], [17, 33]]
    q, k, v, lb, pos, ln, t = _random_cache(d + 7 * with_beta, B, Hq, Hkv, d, cap, lens, with_beta)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.decode_attn(q, k, v, lb, pos, ln, t if with_beta else None)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            g = h // G
            n = ln[b, g]
            bias = None
            if with_beta:
                bias = (t[b] - pos[b, g, :n]).astype(np.float64) * lb[b, g, :n].astype(np.float64)
            eo, el = sdpa_state(f64(q[b, h])[None], f64(k[b, g, :n]), f64(v[b, g, :n]), scale, bias)
            np.testing.assert_allclose(o[b, h], eo[0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], el[0], rtol=0, atol=1e-12)


def test_beta_one_is_plain_attention(oracle):
    q, k, v, _, pos, ln, t = _random_cache(3, 1, 4, 2, 32, 24, [[24, 9]], with_beta=False)
    zeros = np.zeros(pos.shape, np.float32)
    o0, l0 = oracle.decode_attn(q, k, v, None, pos, ln, None)
    o1, l1 = oracle.decode_attn(q, k, v, zeros, pos, ln, t)
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)


@pytest.mark.parametrize("S,split_len", [(1, 0), (2, 0), (7, 0), (64, 0), (5, 8), (10, 3)])
def test_split_states_merge_to_full(oracle, S, split_len):
    """Online-softmax identity (Context Memorization, background): attention over
    a partitioned key set equals the merge of the per-block states."""
    # lengths include multiples of S (28 = 2*14 = 7*4) so the ceil in the split size matters
    q, k, v, lb, pos, ln, t = _random_cache(11, 3, 8, 2, 16, 28, [[27, 13], [1, 0], [28, 14]], True)
    o, lse, op, lp = oracle.decode_attn(q, k, v, lb, pos, ln, t, num_splits=S, split_len=split_len,
                                        want_parts=True)
    B, Hq, _, d = op.shape
    mo, ml = oracle.merge_states(op.transpose(2, 0, 1, 3).reshape(S, B * Hq, d),
                                 lp.transpose(2, 0, 1).reshape(S, B * Hq))
    np.testing.assert_allclose(mo.reshape(B, Hq, d), o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ml.reshape(B, Hq), lse, rtol=0, atol=1e-12)
    # each split is attention over its own contiguous slot range
    scale = 1.0 / math.sqrt(d)
    for b in range(B):
        for h in range(Hq):
            g = h // 4
            n = ln[b, g]
            C = split_len if split_len > 0 else -(-n // S)
            for j in range(S):
                s0, s1 = min(j * C, n), min((j + 1) * C, n)
                if s1 <= s0:
                    assert lp[b, h, j] == -np.inf and not op[b, h, j].any()
                    continue
                bias = (t[b] - pos[b, g, s0:s1]).astype(np.float64) * lb[b, g, s0:s1]
                eo, el = sdpa_state(f64(q[b, h])[None], f64(k[b, g, s0:s1]), f64(v[b, g, s0:s1]), scale, bias)
                np.testing.assert_allclose(op[b, h, j], eo[0], atol=1e-12)
                np.testing.assert_allclose(lp[b, h, j], el[0], atol=1e-12)


def test_split_len_too_small_is_an_error(oracle):
    q, k, v, lb, pos, ln, t = _random_cache(12, 1, 4, 1, 8, 20, [[20]], True)
    with pytest.raises(oracle.OracleError):
        oracle.decode_attn(q, k, v, lb, pos, ln, t, num_splits=2, split_len=8)


def test_gqa_isolation(oracle):
    """Changing kv head g changes exactly query heads g*G .. g*G+G-1."""
    q, k, v, lb, pos, ln, t = _random_cache(5, 1, 8, 4, 16, 12, [[12, 12, 12, 12]], True)
    o0, l0 = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    k2 = k.copy()
    k2[0, 2] = normal_bf16(rng(1), k2[0, 2].shape)
    o1, l1 = oracle.decode_attn(q, k2, v, lb, pos, ln, t)
    changed = np.abs(l1 - l0)[0] > 0
    assert changed.tolist() == [False] * 4 + [True, True] + [False] * 2


def test_empty_and_inactive_rows(oracle):
    q, k, v, lb, pos, ln, t = _random_cache(6, 2, 4, 2, 8, 10, [[0, 10], [10, 10]], True)
    t[1] = -1
    o, lse = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    assert np.all(lse[0, :2] == -np.inf) and not o[0, :2].any()
    assert np.all(np.isfinite(lse[0, 2:]))
    assert np.all(lse[1] == -np.inf) and not o[1].any()


def test_shared_cache_batch_stride_zero(oracle):
    q, k, v, lb, pos, ln, t = _random_cache(7, 3, 4, 2, 16, 30, [[30, 30]] * 3, True)
    k[1:] = k[0]
    v[1:] = v[0]
    lb[1:] = lb[0]
    pos[1:] = pos[0]
    ln = np.array([[5, 9], [30, 1], [17, 30]], np.int32)
    o_full, l_full = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    o_sh, l_sh = oracle.decode_attn(q, k[:1], v[:1], lb[:1], pos[:1], ln, t, kv_batch_stride=0,
                                    meta_batch_stride=0)
    np.testing.assert_array_equal(o_full, o_sh)
    np.testing.assert_array_equal(l_full, l_sh)


def test_default_scale(oracle):
    q, k, v, lb, pos, ln, t = _random_cache(8, 1, 2, 1, 64, 9, [[9]], True)
    a = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    b = oracle.decode_attn(q, k, v, lb, pos, ln, t, scale=1 / 8.0)
    np.testing.assert_array_equal(a[0], b[0])
