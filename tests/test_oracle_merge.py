"""Pins of the oracle's state merge (CPU only): the Z-domain operator of
Context Memorization step 2 as a closed form, the identity element,
commutativity and associativity, and merge of block states == attention over
the union computed by torch SDPA."""
import itertools
import json
import math
import os

import numpy as np
import pytest

from memory_bounded_kv_b200.synth import normal_bf16, rng
from refs import f64, sdpa_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _ev(x):
    return float(eval(str(x), {"__builtins__": {}}, {**vars(math), "inf": math.inf}))


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["merge"], ids=lambda c: c["name"])
def test_closed_forms(oracle, case):
    a = np.array(case["a"], np.float64)[:, None, :]
    l = np.array([_ev(x) for x in case["lse"]])[:, None]
    o, lse = oracle.merge_states(a, l)
    np.testing.assert_allclose(o[0], [_ev(x) for x in case["o"]], atol=1e-14)
    np.testing.assert_allclose(lse[0], _ev(case["lse_out"]), atol=1e-14)


def test_z_domain_formula_random(oracle):
    """(Z_A a_A + Z_B a_B)/(Z_A + Z_B), Z_A + Z_B evaluated literally with moderate Z."""
    g = np.random.default_rng(0)
    for _ in range(50):
        aA, aB = g.normal(size=8), g.normal(size=8)
        ZA, ZB = g.uniform(0.01, 50), g.uniform(0.01, 50)
        o, lse = oracle.merge_states(np.stack([aA, aB])[:, None], np.log([[ZA], [ZB]]))
        np.testing.assert_allclose(o[0], (ZA * aA + ZB * aB) / (ZA + ZB), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(math.exp(lse[0]), ZA + ZB, rtol=1e-13)


def test_empty_merge(oracle):
    o, lse = oracle.merge_states(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(lse == -np.inf) and not o.any()
    o, lse = oracle.merge_states(np.zeros((0, 2, 4)), np.zeros((0, 2)))
    assert np.all(lse == -np.inf) and not o.any()


def test_commutative_associative(oracle):
    g = np.random.default_rng(1)
    n, d = 5, 6
    a = g.normal(size=(n, 1, d))
    l = g.uniform(-30, 30, size=(n, 1))
    ref_o, ref_l = oracle.merge_states(a, l)
    for perm in itertools.permutations(range(n)):
        o, lse = oracle.merge_states(a[list(perm)], l[list(perm)])
        np.testing.assert_allclose(o, ref_o, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, atol=1e-12)
    # ((0,1),(2,3,4)) grouping
    o1, l1 = oracle.merge_states(a[:2], l[:2])
    o2, l2 = oracle.merge_states(a[2:], l[2:])
    o, lse = oracle.merge_states(np.stack([o1, o2]), np.stack([l1, l2]))
    np.testing.assert_allclose(o, ref_o, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, atol=1e-12)


def test_extreme_lse_no_overflow(oracle):
    a = np.array([[[1.0, 2.0]], [[3.0, 4.0]]])
    o, lse = oracle.merge_states(a, np.array([[1000.0], [1000.0 + math.log(3)]]))
    np.testing.assert_allclose(o[0], [2.5, 3.5], atol=1e-12)
    np.testing.assert_allclose(lse[0], 1000.0 + math.log(4), atol=1e-12)


def test_blocks_merge_to_sdpa_over_union(oracle):
    """Online-softmax identity: per-block (a, Z) of attention merged == attention over all keys."""
    g = rng(3, 1)
    d, n = 32, 50
    q = normal_bf16(g, (1, 1, d))
    k = normal_bf16(g, (1, 1, n, d))
    v = normal_bf16(g, (1, 1, n, d))
    pos = np.arange(n, dtype=np.int32)[None, None]
    cuts = [0, 7, 8, 31, 50]
    parts_o, parts_l = [], []
    for s0, s1 in zip(cuts[:-1], cuts[1:]):
        o, l = oracle.decode_attn(q, k[:, :, s0:s1], v[:, :, s0:s1], None, pos[:, :, s0:s1],
                                  np.array([[s1 - s0]], np.int32), None)
        parts_o.append(o.reshape(1, d))
        parts_l.append(l.reshape(1))
    mo, ml = oracle.merge_states(np.stack(parts_o), np.stack(parts_l))
    eo, el = sdpa_state(f64(q[0, 0])[None], f64(k[0, 0]), f64(v[0, 0]), 1 / math.sqrt(d))
    np.testing.assert_allclose(mo[0], eo[0], atol=1e-12)
    np.testing.assert_allclose(ml[0], el[0], atol=1e-12)
