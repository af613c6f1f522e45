"""Pins of the oracle's two-level attention-state-memory lookup (CPU only).

Context Memorization, technical novelty: a hierarchical lookup index brings
retrieval from O(K) to O(log K); expanding the top-16 first-level centroids
matches the linear top-1. Reading: score the C first-level centroids, keep the
m best clusters (the lower cluster on ties), take the argmax over their members
(the lowest entry on ties), merge as the linear lookup does. Pinned against
sklearn's cosine_similarity + numpy's stable argsort (full expansion, coarse
ranking) and against constructed indexes whose answers are known by hand.
"""
import numpy as np

from memory_bounded_kv_b200 import synth
from memory_bounded_kv_b200.synth import to_bf16_bits
from refs import f64, cosine_matrix


def _state(N, H, d, seed=0):
    g = np.random.default_rng(seed)
    return g.standard_normal((N, H, d)).astype(np.float32), g.uniform(1, 4, (N, H)).astype(np.float32)


def test_full_expansion_equals_sklearn_argmax_and_coarse_ranking(oracle):
    w = synth.asm_index_workload(N=12, H=3, K=300, C=17, d=32, seed=11)
    sel, idx, o, lse = oracle.asm_hier_lookup_merge(w.q, w.qhat, w.offsets, w.members, w.qbar, w.abar,
                                                    w.log_zbar, w.o_self, w.lse_self, m=w.C)
    for h in range(w.H):
        qh = f64(w.q[:, h])
        np.testing.assert_array_equal(idx[:, h], np.argmax(cosine_matrix(qh, w.qbar[h]), axis=1))
        coarse = cosine_matrix(qh, w.qhat[h])
        np.testing.assert_array_equal(sel[:, h, :], np.argsort(-coarse, axis=1, kind="stable"))
    idx_l, o_l, lse_l = oracle.asm_lookup_merge(w.q, w.qbar, w.abar, w.log_zbar, w.o_self, w.lse_self)
    np.testing.assert_array_equal(idx, idx_l)
    np.testing.assert_array_equal(o, o_l)
    np.testing.assert_array_equal(lse, lse_l)


def test_partial_expansion_searches_only_the_selected_clusters(oracle):
    """q = e0. Cluster 0 (coarse e0, selected first) holds entry 2 with cos 0.9; cluster 1
    (coarse e1, cos 0) holds entries 0 = e0 (cos 1) and 1 = e1. m = 1 must return 2, m = 2
    the global best 0."""
    d = 8
    e = np.eye(d, dtype=np.float32)
    q = to_bf16_bits(e[0][None, None, :])
    qhat = np.stack([e[0], e[1]])[None]
    qbar = np.stack([e[0], e[1], 0.9 * e[0] + np.sqrt(1 - 0.81) * e[2]]).astype(np.float32)[None]
    offsets = np.array([[0, 1, 3]], np.int32)
    members = np.array([[2, 0, 1]], np.int32)
    abar = to_bf16_bits(np.arange(3 * d, dtype=np.float32).reshape(1, 3, d))
    lz = np.array([[1.0, 2.0, 3.0]], np.float32)
    o_self, l_self = _state(1, 1, d)
    sel, idx, _, _ = oracle.asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m=1)
    assert sel[0, 0].tolist() == [0] and idx[0, 0] == 2
    sel, idx, _, _ = oracle.asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m=2)
    assert sel[0, 0].tolist() == [0, 1] and idx[0, 0] == 0


def test_coarse_ties_select_the_lower_cluster_and_member_ties_the_lowest_entry(oracle):
    """Coarse centroids 0 and 1 are equal: m = 1 keeps cluster 0 (entry 5). With m = 2 the
    same vector also sits at entry 3 of cluster 1: the lower entry wins although its cluster
    was selected second."""
    d = 8
    g = np.random.default_rng(3)
    v = g.standard_normal(d).astype(np.float32)
    q = to_bf16_bits(v[None, None, :])
    qhat = np.stack([v, v, -v])[None].astype(np.float32)
    K = 8
    qbar = g.standard_normal((1, K, d)).astype(np.float32) * 0.01
    qbar[0, 5] = v
    qbar[0, 3] = v
    members = np.array([[5, 0, 3, 1, 2, 4, 6, 7]], np.int32)   # cluster 0: {5, 0}; 1: {3, 1}; 2: rest
    offsets = np.array([[0, 2, 4, 8]], np.int32)
    abar = to_bf16_bits(g.standard_normal((1, K, d)).astype(np.float32))
    lz = np.zeros((1, K), np.float32)
    o_self, l_self = _state(1, 1, d)
    sel, idx, _, _ = oracle.asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m=1)
    assert sel[0, 0].tolist() == [0] and idx[0, 0] == 5
    sel, idx, _, _ = oracle.asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m=2)
    assert sel[0, 0].tolist() == [0, 1] and idx[0, 0] == 3


def test_empty_selected_clusters_leave_the_self_state(oracle):
    d = 8
    e = np.eye(d, dtype=np.float32)
    q = to_bf16_bits(e[0][None, None, :])
    qhat = np.stack([e[0], e[1]])[None]
    qbar = np.stack([e[1], e[2]]).astype(np.float32)[None]
    offsets = np.array([[0, 0, 2]], np.int32)                  # cluster 0 (the best) is empty
    members = np.array([[0, 1]], np.int32)
    abar = to_bf16_bits(np.ones((1, 2, d), np.float32))
    lz = np.array([[4.0, 4.0]], np.float32)
    o_self, l_self = _state(1, 1, d)
    sel, idx, o, lse = oracle.asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m=1)
    assert idx[0, 0] == -1
    np.testing.assert_array_equal(o, o_self.astype(np.float64))
    np.testing.assert_array_equal(lse, l_self.astype(np.float64))
    _, idx, o, lse = oracle.asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m=2)
    assert idx[0, 0] == 0   # cos(e0, e1) = cos(e0, e2) = 0: the lower entry
    assert lse[0, 0] > l_self[0, 0]


def test_m_larger_than_c_and_recall_grows_with_m(oracle):
    w = synth.asm_index_workload(N=16, H=2, K=512, C=16, d=64, seed=12)
    args = (w.q, w.qhat, w.offsets, w.members, w.qbar, w.abar, w.log_zbar, w.o_self, w.lse_self)
    sel, idx_all, _, _ = oracle.asm_hier_lookup_merge(*args, m=40)
    assert (sel[:, :, 16:] == -1).all()
    idx_l, _, _ = oracle.asm_lookup_merge(w.q, w.qbar, w.abar, w.log_zbar, w.o_self, w.lse_self)
    np.testing.assert_array_equal(idx_all, idx_l)
    recall = [(oracle.asm_hier_lookup_merge(*args, m=m)[1] == idx_l).mean() for m in (1, 2, 4, 8, 16)]
    assert all(a <= b for a, b in zip(recall, recall[1:])) and recall[-1] == 1.0
