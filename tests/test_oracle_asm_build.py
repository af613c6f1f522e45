"""Pins of the oracle's attention-state-memory offline build (CPU only).

Context Memorization, core method steps 1-2: the query centroid is the mean of
the cluster's queries; the state centroid folds the members' (a, Z) with the
merge operator, which sums Z. Pinned against: single members (identity), the
page's two-state formula in the Z domain, the pinned n-way merge, the chunked
prefix build (states of one query over disjoint key chunks aggregate to the
SDPA state over all keys, which also fixes Z as a sum), closed-form means, and
a clustering whose answer is known by construction (well-separated groups).
"""
import math

import numpy as np

import oracle.asm_build as ob
from memory_bounded_kv_b200.synth import normal_bf16, rng, to_bf16_bits, bf16_bits_to_f32
from refs import f64, sdpa_state


def _states(g, M, H, d):
    a = g.standard_normal((M, H, d)).astype(np.float32)
    lse = g.uniform(-3, 6, (M, H)).astype(np.float32)
    return a, lse


def test_single_member_is_the_identity_and_empty_is_the_merge_identity():
    g = rng(21, 1)
    M, H, d, K = 3, 2, 16, 5
    q = normal_bf16(g, (M, H, d))
    a, lse = _states(g, M, H, d)
    idx = np.array([[0, 4], [2, 2], [-1, 1]], np.int32)   # row 2 of head 0 belongs to no cluster
    qbar, abar, lz, cnt = ob.asm_aggregate(q, a, lse, idx, K)
    np.testing.assert_array_equal(qbar[0, 0], f64(q[0, 0]))
    np.testing.assert_array_equal(abar[0, 0], a[0, 0].astype(np.float64))
    assert lz[0, 0] == np.float64(lse[0, 0])
    for h, k in ((0, 1), (0, 3), (0, 4), (1, 0), (1, 3)):
        assert cnt[h, k] == 0 and lz[h, k] == -np.inf and not abar[h, k].any() and not qbar[h, k].any()
    assert cnt[0].sum() == 2 and cnt[1].sum() == 3


def test_two_members_follow_the_z_domain_formula():
    g = rng(21, 2)
    d = 8
    q = normal_bf16(g, (2, 1, d))
    a, lse = _states(g, 2, 1, d)
    qbar, abar, lz, _ = ob.asm_aggregate(q, a, lse, np.zeros((2, 1), np.int32), 1)
    za, zb = math.exp(lse[0, 0]), math.exp(lse[1, 0])
    expect = (za * a[0, 0].astype(np.float64) + zb * a[1, 0].astype(np.float64)) / (za + zb)
    np.testing.assert_allclose(abar[0, 0], expect, rtol=1e-13, atol=1e-14)
    assert abs(lz[0, 0] - math.log(za + zb)) < 1e-13
    np.testing.assert_allclose(qbar[0, 0], (f64(q[0, 0]) + f64(q[1, 0])) / 2, rtol=0, atol=0)


def test_fold_equals_the_pinned_n_way_merge_in_any_order(oracle):
    g = rng(21, 3)
    M, d = 9, 32
    q = normal_bf16(g, (M, 1, d))
    a, lse = _states(g, M, 1, d)
    lse[3, 0] = -np.inf            # a member with an empty prefix contributes nothing
    qbar, abar, lz, _ = ob.asm_aggregate(q, a, lse, np.zeros((M, 1), np.int32), 1)
    for perm in (np.arange(M), g.permutation(M)):
        o, l = oracle.merge_states(a[perm, 0][:, None, :], lse[perm, 0][:, None])
        np.testing.assert_allclose(abar[0, 0], o[0], rtol=1e-12, atol=1e-13)
        assert abs(lz[0, 0] - l[0]) < 1e-12


def test_chunked_prefix_build_equals_attention_over_the_whole_prefix():
    """One query's states over 4 disjoint key chunks, aggregated as one cluster, equal its state
    over the union of the chunks (the chunked prefix build of the page): Z must be summed."""
    g = rng(21, 4)
    d, P = 64, 4 * 250
    scale = 1 / math.sqrt(d)
    qv = normal_bf16(g, (1, d))
    k, v = normal_bf16(g, (P, d)), normal_bf16(g, (P, d))
    parts = [sdpa_state(f64(qv), f64(k[j * 250:(j + 1) * 250]), f64(v[j * 250:(j + 1) * 250]), scale)
             for j in range(4)]
    a = np.stack([p[0][0] for p in parts])[:, None, :]
    lse = np.array([p[1][0] for p in parts])[:, None]
    q = np.repeat(qv[None], 4, axis=0)
    _, abar, lz, _ = ob.asm_aggregate(q, a, lse, np.zeros((4, 1), np.int32), 1)
    eo, el = sdpa_state(f64(qv), f64(k), f64(v), scale)
    np.testing.assert_allclose(abar[0, 0], eo[0], rtol=1e-10, atol=1e-12)
    assert abs(lz[0, 0] - el[0]) < 1e-10
    _, _, lz_mean, _ = ob.asm_aggregate(q, a, lse, np.zeros((4, 1), np.int32), 1, z_mean=True)
    assert abs(lz_mean[0, 0] - (el[0] - math.log(4))) < 1e-10


def test_query_centroid_closed_forms():
    d = 16
    x = np.linspace(-2, 2, d).astype(np.float32)
    q = to_bf16_bits(np.stack([x, x, -x, x * 0.5, x * 1.5])[:, None, :])
    idx = np.array([[0], [0], [1], [1], [2]], np.int32)
    idx[2, 0] = 1
    idx[3, 0] = 3
    idx[4, 0] = 3
    qbar, abar, lz, cnt = ob.asm_aggregate(q, None, None, idx, 4)
    xb = bf16_bits_to_f32(to_bf16_bits(x)).astype(np.float64)
    np.testing.assert_array_equal(qbar[0, 0], xb)                 # {x, x}
    np.testing.assert_array_equal(qbar[0, 1], -xb)                # {-x}
    assert not qbar[0, 2].any() and cnt[0, 2] == 0                # empty
    np.testing.assert_allclose(qbar[0, 3], xb, rtol=1e-2)          # {x/2, 3x/2} (bf16 inputs)
    assert abar is None and lz is None


def _separated(g, M, H, K, d, spread=0.05):
    """K groups per head around random unit directions, a small spread: group membership is the
    nearest direction by a wide margin."""
    u = g.standard_normal((H, K, d))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    owner = np.stack([g.permutation(np.arange(M) % K) for _ in range(H)], axis=1)   # [M, H]
    x = u[np.arange(H)[None, :], owner] + spread * g.standard_normal((M, H, d))
    return to_bf16_bits(x.astype(np.float32)), owner.astype(np.int32)


def test_kmeans_recovers_separated_groups_and_never_loses_objective():
    g = rng(21, 6)
    M, H, K, d = 96, 2, 6, 32
    q, owner = _separated(g, M, H, K, d)
    init = np.stack([np.array([np.nonzero(owner[:, h] == k)[0][0] for k in range(K)]) for h in range(H)])
    idx, cent = ob.asm_kmeans(q, init, iters=3)
    np.testing.assert_array_equal(idx, owner)            # the groups, numbered by their first member
    qf = f64(q)
    obj = []
    idx_t = ob.cosine_assign(q, np.stack([qf[init[h], h] for h in range(H)]))
    for _ in range(4):
        c, _, _, _ = ob.asm_aggregate(q, None, None, idx_t, K)
        cn = c / np.maximum(np.linalg.norm(c, axis=-1, keepdims=True), 1e-300)
        obj.append(sum((qf[:, h] * cn[h, idx_t[:, h]]).sum() for h in range(H)))
        idx_t = ob.cosine_assign(q, c)
    assert all(b >= a - 1e-9 for a, b in zip(obj, obj[1:]))


def test_kmeans_from_a_poor_start_still_improves():
    """Two initial centroids in the same group: Lloyd moves one of them; the objective rises."""
    g = rng(21, 7)
    M, H, K, d = 60, 1, 3, 16
    q, owner = _separated(g, M, H, K, d, spread=0.2)
    g0 = np.nonzero(owner[:, 0] == 0)[0]
    g2 = np.nonzero(owner[:, 0] == 2)[0]
    init = np.array([[g0[0], g0[1], g2[0]]])
    qf = f64(q)
    c0 = qf[init[0], 0][None]
    idx0 = ob.cosine_assign(q, c0)
    idx, cent = ob.asm_kmeans(q, init, iters=5)

    def objective(ix):
        c, _, _, _ = ob.asm_aggregate(q, None, None, ix, K)
        cn = c / np.maximum(np.linalg.norm(c, axis=-1, keepdims=True), 1e-300)
        return (qf[:, 0] * cn[0, ix[:, 0]]).sum()
    assert objective(idx) >= objective(idx0)


def test_index_of_a_clustered_memory_lists_each_group_once(oracle):
    """Entries scattered around C directions: the index recovers the groups (entries listed in
    increasing order), and the two-level lookup with every cluster kept equals the linear one."""
    g = rng(21, 8)
    H, C, per, d = 2, 5, 12, 32
    K = C * per
    u = g.standard_normal((H, C, d))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    owner = np.stack([g.permutation(np.arange(K) % C) for _ in range(H)])          # [H, K]
    qbar = (u[np.arange(H)[:, None], owner] + 0.05 * g.standard_normal((H, K, d))).astype(np.float32)
    init = np.stack([np.array([np.nonzero(owner[h] == c)[0][0] for c in range(C)]) for h in range(H)])
    qhat, offsets, members, idx = ob.asm_index(qbar, init, iters=2)
    for h in range(H):
        np.testing.assert_array_equal(idx[:, h], owner[h])
        for c in range(C):
            np.testing.assert_array_equal(members[h, offsets[h, c]:offsets[h, c + 1]], np.nonzero(owner[h] == c)[0])
        assert offsets[h, -1] == K
    q = normal_bf16(g, (4, H, d))
    abar = normal_bf16(g, (H, K, d))
    lz = g.uniform(1, 3, (H, K)).astype(np.float32)
    o_self, l_self = g.standard_normal((4, H, d)).astype(np.float32), np.zeros((4, H), np.float32)
    _, idx_h, _, _ = oracle.asm_hier_lookup_merge(q, qhat.astype(np.float32), offsets, members, qbar, abar, lz,
                                                  o_self, l_self, C)
    idx_l, _, _ = oracle.asm_lookup_merge(q, qbar, abar, lz, o_self, l_self)
    np.testing.assert_array_equal(idx_h, idx_l)


def test_group_helpers_route_rows_and_tables():
    x = np.arange(3 * 4 * 2).reshape(3, 4, 2)           # M = 3, H = 4 heads
    y = ob.group_rows(x, 2)                              # 2 tables of 2 heads
    assert y.shape == (6, 2, 2)
    for i in range(3):
        for h in range(4):
            hits = [r for r in range(6) if (y[r, h // 2] == x[i, h]).all()]
            assert len(hits) == 1 and hits[0] // 2 == i
    t = np.arange(2 * 3).reshape(2, 3)
    np.testing.assert_array_equal(ob.expand_tables(t, 2), t[[0, 0, 1, 1]])


def test_assignment_ties_and_zero_vectors_take_the_lower_index():
    d = 8
    v = np.linspace(0.5, 1.5, d).astype(np.float32)
    q = to_bf16_bits(np.stack([v, np.zeros(d, np.float32)])[:, None, :])   # a query, a zero query
    cent = np.stack([-v, v, v, 2 * v])[None].astype(np.float64)            # entries 1, 2, 3 tie at cos 1
    idx = ob.cosine_assign(q, cent)
    assert idx[0, 0] == 1 and idx[1, 0] == 0


def test_one_lloyd_step_moves_a_centroid_by_hand():
    """Unit vectors at 0, 10, 80 and 90 degrees; centroids start at the first two. Assignment:
    [0, 1, 1, 1] (80 and 90 are nearer 10 than 0). Update: centroid 1 = mean of 10, 80, 90 degrees
    (about 60 degrees). Reassignment: 10 degrees is now nearer 0 -> [0, 0, 1, 1]."""
    ang = np.deg2rad([0.0, 10.0, 80.0, 90.0])
    x = np.zeros((4, 1, 16), np.float32)
    x[:, 0, 0], x[:, 0, 1] = np.cos(ang), np.sin(ang)
    q = to_bf16_bits(x)
    init = np.array([[0, 1]])
    idx0, _ = ob.asm_kmeans(q, init, iters=0)
    idx1, cent = ob.asm_kmeans(q, init, iters=1)
    np.testing.assert_array_equal(idx0[:, 0], [0, 1, 1, 1])
    np.testing.assert_array_equal(idx1[:, 0], [0, 0, 1, 1])
    c1 = cent[0, 1, :2]
    assert 55 < np.rad2deg(np.arctan2(c1[1], c1[0])) < 65
