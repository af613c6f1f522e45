"""Pins of the oracle's attention-state-memory lookup and merge (CPU only).

Context Memorization, core method steps 3-4: c* = argmax_k cos(q, qbar_k),
then merge of the retrieved (abar, Zbar) with the query's own attention, which
the page calls lossless by the online-softmax identity. Pinned against
sklearn's cosine_similarity, exact-match retrieval (K = number of calibration
queries, qbar_k = q_k / |q_k|), and merged state == SDPA over prefix + self.
"""
import math

import numpy as np

from memory_bounded_kv_b200.synth import normal_bf16, rng, to_bf16_bits, bf16_bits_to_f32
from refs import f64, sdpa_state, cosine_matrix


def test_argmax_matches_sklearn(oracle):
    g = rng(4, 7)
    N, H, K, d = 6, 3, 200, 16
    q = normal_bf16(g, (N, H, d))
    qbar = g.standard_normal((H, K, d)).astype(np.float32)
    abar = normal_bf16(g, (H, K, d))
    lz = g.uniform(5, 12, (H, K)).astype(np.float32)
    o_self = g.standard_normal((N, H, d)).astype(np.float32)
    l_self = g.uniform(0, 3, (N, H)).astype(np.float32)
    idx, o, lse = oracle.asm_lookup_merge(q, qbar, abar, lz, o_self, l_self)
    for h in range(H):
        cos = cosine_matrix(f64(q[:, h]), qbar[h])
        np.testing.assert_array_equal(idx[:, h], np.argmax(cos, axis=1))
        for n in range(N):
            np.testing.assert_allclose(oracle.asm_cosines(q, qbar, n, h), cos[n], atol=1e-12)


def test_exact_match_retrieves_own_entry(oracle):
    g = rng(4, 8)
    N, H, d = 64, 2, 32
    q = normal_bf16(g, (N, H, d))
    qbar = np.stack([f64(q[:, h]) / np.linalg.norm(f64(q[:, h]), axis=1, keepdims=True) for h in range(H)])
    idx, _, _ = oracle.asm_lookup_merge(q, qbar.astype(np.float32), normal_bf16(g, (H, N, d)),
                                        np.zeros((H, N), np.float32), np.zeros((N, H, d), np.float32),
                                        np.zeros((N, H), np.float32))
    np.testing.assert_array_equal(idx, np.tile(np.arange(N)[:, None], (1, H)))


def test_merge_with_stored_prefix_state_is_lossless(oracle):
    """Stored (abar, log Zbar) = attention state of q over a prefix; merging it with
    the self state equals attention over prefix + self (up to bf16 storage of abar)."""
    g = rng(4, 9)
    d, P, L = 64, 300, 40
    scale = 1 / math.sqrt(d)
    q = normal_bf16(g, (1, 1, d))
    kp, vp = normal_bf16(g, (P, d)), normal_bf16(g, (P, d))
    ks, vs = normal_bf16(g, (1, 1, L, d)), normal_bf16(g, (1, 1, L, d))
    a_pref, l_pref = sdpa_state(f64(q[0, 0])[None], f64(kp), f64(vp), scale)
    o_self, l_self = oracle.decode_attn(q, ks, vs, None, np.arange(L, dtype=np.int32)[None, None],
                                        np.array([[L]], np.int32), None)
    qbar = (f64(q[0, 0]) / np.linalg.norm(f64(q[0, 0])))[None, None].astype(np.float32)
    abar = to_bf16_bits(a_pref.astype(np.float32))[None]
    idx, o, lse = oracle.asm_lookup_merge(q, qbar, abar, l_pref.astype(np.float32)[None],
                                          o_self.astype(np.float32), l_self.astype(np.float32))
    eo, el = sdpa_state(f64(q[0, 0])[None], np.concatenate([f64(kp), f64(ks[0, 0])]),
                        np.concatenate([f64(vp), f64(vs[0, 0])]), scale)
    assert idx[0, 0] == 0
    # abar is stored as bf16: error bounded by its rounding (2^-9 relative)
    np.testing.assert_allclose(o[0, 0], eo[0], atol=4e-3 * np.abs(a_pref).max() + 1e-6)
    np.testing.assert_allclose(lse[0, 0], el[0], atol=1e-6)
    # with the stored state exactly representable the merge is exact
    abar_exact = bf16_bits_to_f32(abar).astype(np.float64)[0, 0]
    z_p, z_s = math.exp(l_pref[0]), math.exp(l_self[0, 0])
    expect = (z_p * abar_exact + z_s * o_self[0, 0].astype(np.float32)) / (z_p + z_s)
    np.testing.assert_allclose(o[0, 0], expect, atol=1e-6)


def test_zero_norm_query_picks_first_entry(oracle):
    N, H, K, d = 1, 1, 5, 8
    q = np.zeros((N, H, d), np.uint16)
    qbar = rng(1).standard_normal((H, K, d)).astype(np.float32)
    idx, _, _ = oracle.asm_lookup_merge(q, qbar, np.zeros((H, K, d), np.uint16), np.zeros((H, K), np.float32),
                                        np.zeros((N, H, d), np.float32), np.zeros((N, H), np.float32))
    assert idx[0, 0] == 0
