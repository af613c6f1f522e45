"""GPU parity of kvb_asm_hier_lookup_merge (two-level attention-state-memory
lookup) against the oracle: clustered memories with ragged clusters and
scattered entry ids, partial and full expansion, m > C, hand-built indexes
(best entry outside the selected clusters, ties, empty clusters), bad member
ids, and the 32-head / 4096-entry / 64-cluster / top-16 case the bench times."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200 import synth
from memory_bounded_kv_b200.synth import to_bf16_bits
from gpu_util import dev, host, assert_state_close

pytestmark = pytest.mark.gpu

TIE = 1e-6   # cosines closer than this may be ordered either way (fp32 scores vs fp64 oracle)


def run_hier(q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m):
    N, H, d = q.shape
    idx = torch.full((N, H), -7, dtype=torch.int32, device="cuda")
    o = torch.zeros(N, H, d, device="cuda")
    lse = torch.zeros(N, H, device="cuda")
    ws = torch.empty(kvb.kvb_asm_hier_workspace_bytes(N, H, m), dtype=torch.uint8, device="cuda")
    kvb.kvb_asm_hier_lookup_merge(dev(q), dev(qhat), dev(offsets), dev(members), dev(qbar), dev(abar), dev(lz),
                                  dev(o_self), dev(l_self), idx, o, lse, ws, m)
    torch.cuda.synchronize()
    nhm = N * H * m
    sel = host(ws[nhm * 8: nhm * 12].view(torch.int32)).reshape(N, H, m)
    return sel, host(idx), host(o), host(lse)


def check_hier(oracle, q, qhat, offsets, members, qbar, abar, lz, o_self, l_self, m, sel, idx, o, lse):
    """sel: the oracle's clusters, or a set that differs only at a first-level near tie.
    idx: the exact best (lowest entry among equal cosines) over the clusters the GPU selected,
    or a near tie of it. (o, lse): the oracle's merge with the GPU's entry."""
    sel_r, idx_r, o_r, lse_r = oracle.asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, lz, o_self,
                                                            l_self, m)
    N, H, d = q.shape
    C = qhat.shape[1]
    mm = min(m, C)
    assert (sel[:, :, mm:] == -1).all()
    explained = 0
    for n in range(N):
        for h in range(H):
            if (sel[n, h] == sel_r[n, h]).all() and idx[n, h] == idx_r[n, h]:
                continue
            explained += 1
            coarse = oracle.asm_cosines(q, qhat, n, h)
            g_set, r_set = set(sel[n, h, :mm].tolist()), set(sel_r[n, h, :mm].tolist())
            if g_set != r_set:   # boundary of the top-m: the swapped clusters tie
                lo = min(coarse[c] for c in g_set)
                hi = max(coarse[c] for c in set(range(C)) - g_set)
                assert hi - lo <= TIE, (n, h, sorted(g_set), sorted(r_set))
            cos = oracle.asm_cosines(q, qbar, n, h)
            cand = [int(k) for c in sel[n, h, :mm] for k in members[h, offsets[h, c]:offsets[h, c + 1]]]
            if not cand:
                assert idx[n, h] == -1
                continue
            best = min(cand, key=lambda k: (-cos[k], k))
            assert idx[n, h] in cand and cos[best] - cos[idx[n, h]] <= TIE, (n, h, idx[n, h], best)
            one = oracle.asm_lookup_merge(q[n:n + 1, h:h + 1], qbar[h:h + 1, idx[n, h]:idx[n, h] + 1],
                                          abar[h:h + 1, idx[n, h]:idx[n, h] + 1], lz[h:h + 1, idx[n, h]:idx[n, h] + 1],
                                          o_self[n:n + 1, h:h + 1], l_self[n:n + 1, h:h + 1])
            o_r[n, h], lse_r[n, h] = one[1][0, 0], one[2][0, 0]
    assert_state_close(o, lse, o_r, lse_r, "hierarchical merge")
    return explained


def _args(w):
    return (w.q, w.qhat, w.offsets, w.members, w.qbar, w.abar, w.log_zbar, w.o_self, w.lse_self)


@pytest.mark.parametrize("N,H,K,C,m", [(4, 3, 500, 23, 4), (5, 2, 300, 17, 17), (3, 2, 130, 8, 20),
                                       (9, 1, 64, 1, 1), (7, 4, 1000, 31, 1), (2, 2, 3000, 1024, 64)])
def test_hier_matches_oracle(oracle, N, H, K, C, m):
    w = synth.asm_index_workload(N=N, H=H, K=K, C=C, seed=N * 100 + C)
    sel, idx, o, lse = run_hier(*_args(w), m)
    assert check_hier(oracle, *_args(w), m, sel, idx, o, lse) <= max(1, N * H // 50)


def test_full_expansion_equals_linear_lookup(oracle):
    w = synth.asm_index_workload(N=6, H=3, K=700, C=12, seed=5)
    sel, idx, o, lse = run_hier(*_args(w), 12)
    idx_l = torch.zeros(6, 3, dtype=torch.int32, device="cuda")
    o_l = torch.zeros(6, 3, 128, device="cuda")
    lse_l = torch.zeros(6, 3, device="cuda")
    ws = torch.empty(kvb.kvb_asm_workspace_bytes(6, 3, 700), dtype=torch.uint8, device="cuda")
    kvb.kvb_asm_lookup_merge(dev(w.q), dev(w.qbar), dev(w.abar), dev(w.log_zbar), dev(w.o_self), dev(w.lse_self),
                             idx_l, o_l, lse_l, ws)
    check_hier(oracle, *_args(w), 12, sel, idx, o, lse)
    same = idx == host(idx_l)
    cos_ok = all(abs(oracle.asm_cosines(w.q, w.qbar, n, h)[idx[n, h]] -
                     oracle.asm_cosines(w.q, w.qbar, n, h)[host(idx_l)[n, h]]) <= TIE
                 for n, h in np.argwhere(~same))
    assert cos_ok


def test_constructed_indexes(oracle):
    """Best entry outside the selected cluster (m = 1 -> 2, m = 2 -> 0), equal first-level
    centroids (lower cluster), equal entries (lower id), an empty best cluster (self state)."""
    d = 128
    e = np.eye(d, dtype=np.float32)
    o_self = np.random.default_rng(0).standard_normal((1, 1, d)).astype(np.float32)
    l_self = np.array([[2.5]], np.float32)
    q = to_bf16_bits(e[0][None, None, :])
    qhat = np.stack([e[0], e[1]])[None]
    qbar = np.stack([e[0], e[1], 0.9 * e[0] + np.sqrt(1 - 0.81) * e[2]]).astype(np.float32)[None]
    abar = to_bf16_bits(np.arange(3 * d, dtype=np.float32).reshape(1, 3, d) / 100)
    lz = np.array([[1.0, 2.0, 3.0]], np.float32)
    for m, want in ((1, 2), (2, 0)):
        args = (q, qhat, np.array([[0, 1, 3]], np.int32), np.array([[2, 0, 1]], np.int32), qbar, abar, lz,
                o_self, l_self)
        sel, idx, o, lse = run_hier(*args, m)
        assert idx[0, 0] == want
        check_hier(oracle, *args, m, sel, idx, o, lse)
    # ties: clusters 0 and 1 share a first-level centroid; entries 5 and 3 are the same vector
    g = np.random.default_rng(3)
    v = g.standard_normal(d).astype(np.float32)
    v16 = (to_bf16_bits(v).astype(np.uint32) << 16).view(np.float32)
    K = 8
    qbar = (g.standard_normal((1, K, d)) * 0.01).astype(np.float32)
    qbar[0, 5] = qbar[0, 3] = v16
    args = (to_bf16_bits(v16[None, None, :]), np.stack([v16, v16, -v16])[None].astype(np.float32),
            np.array([[0, 2, 4, 8]], np.int32), np.array([[5, 0, 3, 1, 2, 4, 6, 7]], np.int32), qbar,
            to_bf16_bits(g.standard_normal((1, K, d)).astype(np.float32)), np.zeros((1, K), np.float32),
            o_self, l_self)
    for m, want in ((1, 5), (2, 3)):
        sel, idx, o, lse = run_hier(*args, m)
        assert sel[0, 0, 0] == 0 and idx[0, 0] == want
        check_hier(oracle, *args, m, sel, idx, o, lse)
    # the best cluster is empty: nothing retrieved with m = 1
    args = (q, np.stack([e[0], e[1]])[None], np.array([[0, 0, 2]], np.int32), np.array([[0, 1]], np.int32),
            np.stack([e[1], e[2]]).astype(np.float32)[None], to_bf16_bits(np.ones((1, 2, d), np.float32)),
            np.array([[4.0, 4.0]], np.float32), o_self, l_self)
    sel, idx, o, lse = run_hier(*args, 1)
    assert idx[0, 0] == -1
    np.testing.assert_array_equal(o, o_self)
    np.testing.assert_array_equal(lse, l_self)


def test_bad_member_ids_set_the_range_error():
    w = synth.asm_index_workload(N=2, H=2, K=200, C=4, seed=9)
    w.members[1, 3] = 200      # out of range
    w.members[0, 0] = -1
    kvb.kvb_get_error()
    run_hier(*_args(w), 4)
    assert kvb.kvb_get_error() & 4
    assert kvb.kvb_get_error() == 0


def test_bench_shape_parity_and_recall(oracle):
    """32 heads, 4096 entries, 64 clusters, top-16; 16 query tokens."""
    w = synth.asm_index_workload(N=16, H=32, K=4096, C=64)
    sel, idx, o, lse = run_hier(*_args(w), 16)
    assert check_hier(oracle, *_args(w), 16, sel, idx, o, lse) <= 5
    idx_l, _, _ = oracle.asm_lookup_merge(w.q, w.qbar, w.abar, w.log_zbar, w.o_self, w.lse_self)
    assert (idx == idx_l).mean() >= 0.9
