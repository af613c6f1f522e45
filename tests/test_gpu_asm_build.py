"""GPU parity of the attention-state-memory offline build against the oracle:
kvb_asm_aggregate (ragged and empty clusters, unassigned queries, members with
Z = 0, sum and mean Z, queries only), the range error, the cosine Lloyd
clustering on separated groups, and the whole build (clusters + aggregation)."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200 import asm_build
from memory_bounded_kv_b200.synth import normal_bf16, rng, to_bf16_bits
import oracle.asm_build as ob
from gpu_util import dev, host, assert_state_close, bf16_round

pytestmark = pytest.mark.gpu


def run_aggregate(q, a, lse, idx, K, z_mean=False):
    M, H, d = q.shape
    qbar = torch.full((H, K, d), 7.0, device="cuda")
    abar = torch.zeros(H, K, d, dtype=torch.bfloat16, device="cuda")
    lz = torch.zeros(H, K, device="cuda")
    cnt = torch.full((H, K), -5, dtype=torch.int32, device="cuda")
    ws = torch.empty(kvb.kvb_asm_aggregate_workspace_bytes(H, K), dtype=torch.uint8, device="cuda")
    with_states = a is not None
    kvb.kvb_asm_aggregate(dev(q), dev(a) if with_states else None, dev(lse) if with_states else None, dev(idx),
                          qbar, abar if with_states else None, lz if with_states else None, cnt, ws,
                          z_mean=z_mean)
    torch.cuda.synchronize()
    return host(qbar), host(abar.float()), host(lz), host(cnt)


def check_aggregate(got, want, with_states=True):
    qbar, abar, lz, cnt = got
    q_r, a_r, l_r, c_r = want
    np.testing.assert_array_equal(cnt, c_r)
    np.testing.assert_allclose(qbar, q_r, rtol=1e-5, atol=1e-6)
    if with_states:
        H, K, d = a_r.shape
        assert_state_close(abar.reshape(H * K, d), lz.reshape(-1), bf16_round(a_r).reshape(H * K, d),
                           l_r.reshape(-1), "aggregated state")


def _inputs(seed, M, H, K, d=128):
    g = rng(seed, 31)
    q = normal_bf16(g, (M, H, d))
    a = g.standard_normal((M, H, d)).astype(np.float32)
    lse = g.uniform(-4, 9, (M, H)).astype(np.float32)
    lse[g.random((M, H)) < 0.03] = -np.inf                  # members with an empty prefix
    idx = g.integers(-1, K, (M, H)).astype(np.int32)          # -1: in no cluster
    idx[:, 0] = np.where(idx[:, 0] == 3, 4, idx[:, 0])        # cluster 3 of head 0 stays empty
    return q, a, lse, idx


@pytest.mark.parametrize("M,H,K", [(500, 3, 37), (64, 1, 1), (2000, 2, 300)])
@pytest.mark.parametrize("z_mean", [False, True])
def test_aggregate_matches_oracle(M, H, K, z_mean):
    q, a, lse, idx = _inputs(M + K, M, H, K)
    got = run_aggregate(q, a, lse, idx, K, z_mean)
    want = ob.asm_aggregate(q, a, lse, idx, K, z_mean)
    check_aggregate(got, want)


def test_cluster_of_empty_prefixes_is_the_merge_identity():
    q, a, lse, idx = _inputs(5, 40, 1, 4)
    idx[:, 0] = np.arange(40) % 4
    lse[idx[:, 0] == 2, 0] = -np.inf
    got = run_aggregate(q, a, lse, idx, 4)
    assert got[2][0, 2] == -np.inf and not got[1][0, 2].any() and got[3][0, 2] == 10
    check_aggregate(got, ob.asm_aggregate(q, a, lse, idx, 4))


def test_queries_only():
    q, a, lse, idx = _inputs(6, 300, 2, 11)
    got = run_aggregate(q, None, None, idx, 11)
    want = ob.asm_aggregate(q, None, None, idx, 11)
    check_aggregate(got, want, with_states=False)


def test_cluster_out_of_range_sets_the_range_error():
    q, a, lse, idx = _inputs(7, 50, 1, 5)
    idx[3, 0] = 5
    kvb.kvb_get_error()
    got = run_aggregate(q, a, lse, idx, 5)
    assert kvb.kvb_get_error() & 4
    idx_ok = idx.copy()
    idx_ok[3, 0] = -1
    check_aggregate(got, ob.asm_aggregate(q, a, lse, idx_ok, 5))


def _separated(seed, M, H, K, d=128, spread=0.05):
    g = rng(seed, 32)
    u = g.standard_normal((H, K, d))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    owner = np.stack([g.permutation(np.arange(M) % K) for _ in range(H)], axis=1)
    x = u[np.arange(H)[None, :], owner] + spread * g.standard_normal((M, H, d))
    init = np.stack([np.array([np.nonzero(owner[:, h] == k)[0][0] for k in range(K)]) for h in range(H)])
    return to_bf16_bits(x.astype(np.float32)), owner.astype(np.int32), init


def test_kmeans_matches_oracle_on_separated_groups():
    q, owner, init = _separated(8, 384, 2, 12)
    idx, cent = asm_build.asm_kmeans(dev(q), init, iters=3)
    idx_r, cent_r = ob.asm_kmeans(q, init, iters=3)
    np.testing.assert_array_equal(idx_r, owner)
    np.testing.assert_array_equal(host(idx), idx_r)
    np.testing.assert_allclose(host(cent), cent_r, rtol=1e-5, atol=1e-6)


def test_kmeans_from_overlapping_starts_matches_oracle():
    """Wider groups and two starting centroids in one group: the clusters move over the
    iterations; every assignment on the way must match the oracle's (margins checked)."""
    q, owner, init = _separated(9, 256, 1, 8, spread=0.3)
    init[0, 1] = np.nonzero(owner[:, 0] == 0)[0][1]
    idx, cent = asm_build.asm_kmeans(dev(q), init, iters=4)
    idx_r, cent_r = ob.asm_kmeans(q, init, iters=4)
    # the oracle's decisions must not sit on a near tie for the comparison to be exact
    qf = (q.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    cn = cent_r / np.maximum(np.linalg.norm(cent_r, axis=-1, keepdims=True), 1e-300)
    cos = np.einsum("md,kd->mk", qf[:, 0] / np.linalg.norm(qf[:, 0], axis=1, keepdims=True), cn[0])
    top = np.sort(cos, axis=1)
    assert (top[:, -1] - top[:, -2]).min() > 1e-4
    np.testing.assert_array_equal(host(idx), idx_r)
    np.testing.assert_allclose(host(cent), cent_r, rtol=1e-5, atol=1e-6)


def test_build_matches_oracle():
    q, owner, init = _separated(10, 320, 2, 10)
    g = rng(10, 33)
    a = g.standard_normal(q.shape).astype(np.float32)
    lse = g.uniform(0, 8, q.shape[:2]).astype(np.float32)
    qbar, abar, lz, cnt, idx = asm_build.asm_build(dev(q), dev(a), dev(lse), init, iters=2)
    idx_r, _ = ob.asm_kmeans(q, init, iters=2)
    np.testing.assert_array_equal(host(idx), idx_r)
    want = ob.asm_aggregate(q, a, lse, idx_r, 10)
    check_aggregate((host(qbar), host(abar.float()), host(lz), host(cnt)), want)


def test_index_build_matches_oracle_and_serves_the_two_level_lookup(oracle):
    """A memory whose entries sit in 16 groups per head: the GPU index (bf16 entries clustered
    by the lookup + mean update, then the deterministic cluster lists) equals the oracle's, and
    the two-level lookup through it answers as the oracle's lookup through the oracle's index."""
    from test_gpu_asm_hier import run_hier, check_hier
    g = rng(11, 34)
    H, C, per, d = 3, 16, 40, 128
    K = C * per
    u = g.standard_normal((H, C, d))
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    owner = np.stack([g.permutation(np.arange(K) % C) for _ in range(H)])             # [H, K]
    qbar = (u[np.arange(H)[:, None], owner] + 0.05 * g.standard_normal((H, K, d))).astype(np.float32)
    init = np.stack([np.array([np.nonzero(owner[h] == c)[0][0] for c in range(C)]) for h in range(H)])
    qhat, offsets, members, idx = asm_build.asm_index(dev(qbar), init, iters=2)
    qhat_r, off_r, mem_r, idx_r = ob.asm_index(qbar, init, 2)
    np.testing.assert_array_equal(idx_r, owner.T)
    np.testing.assert_array_equal(host(idx), idx_r)
    np.testing.assert_array_equal(host(offsets), off_r)
    np.testing.assert_array_equal(host(members), mem_r)
    np.testing.assert_allclose(host(qhat), qhat_r, rtol=1e-5, atol=1e-6)
    N, m = 24, 4
    q = normal_bf16(g, (N, H, d))
    abar = normal_bf16(g, (H, K, d))
    lz = g.uniform(2, 9, (H, K)).astype(np.float32)
    o_self = g.standard_normal((N, H, d)).astype(np.float32)
    l_self = g.uniform(1, 5, (N, H)).astype(np.float32)
    sel, hidx, o, lse = run_hier(q, host(qhat), host(offsets), host(members), qbar, abar, lz, o_self, l_self, m)
    check_hier(oracle, q, qhat_r.astype(np.float32), off_r, mem_r, qbar, abar, lz, o_self, l_self, m,
               sel, hidx, o, lse)


def test_grouped_lookup_reads_the_group_table(oracle):
    """8 query heads sharing 2 tables (GQA groups of 4): equal to the per-head lookup with each
    head given its group's table."""
    from test_gpu_kernels import check_asm
    g = rng(12, 35)
    N, H, Ht, K, d = 50, 8, 2, 300, 128
    q = normal_bf16(g, (N, H, d))
    x = g.standard_normal((Ht, K, d))
    qbar = (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)
    abar = normal_bf16(g, (Ht, K, d))
    lz = g.uniform(5, 12, (Ht, K)).astype(np.float32)
    o_self = g.standard_normal((N, H, d)).astype(np.float32)
    l_self = g.uniform(3, 9, (N, H)).astype(np.float32)
    idx = torch.zeros(N, H, dtype=torch.int32, device="cuda")
    o = torch.zeros(N, H, d, device="cuda")
    lse = torch.zeros(N, H, device="cuda")
    ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, K), dtype=torch.uint8, device="cuda")
    kvb.kvb_asm_lookup_merge_grouped(dev(q), dev(qbar), dev(abar), dev(lz), dev(o_self), dev(l_self), idx, o, lse, ws)
    torch.cuda.synchronize()
    G = H // Ht
    check_asm(oracle, q, ob.expand_tables(qbar, G), ob.expand_tables(abar, G), ob.expand_tables(lz, G), o_self,
              l_self, host(idx), host(o), host(lse))


def test_grouped_aggregate_folds_the_group_rows():
    q, a, lse, idx = _inputs(13, 200, 8, 23)
    Ht, G, K = 2, 4, 23
    qbar = torch.zeros(Ht, K, 128, device="cuda")
    abar = torch.zeros(Ht, K, 128, dtype=torch.bfloat16, device="cuda")
    lz = torch.zeros(Ht, K, device="cuda")
    cnt = torch.zeros(Ht, K, dtype=torch.int32, device="cuda")
    ws = torch.empty(kvb.kvb_asm_aggregate_workspace_bytes(Ht, K), dtype=torch.uint8, device="cuda")
    kvb.kvb_asm_aggregate_grouped(dev(q), dev(a), dev(lse), dev(idx), qbar, abar, lz, cnt, ws)
    torch.cuda.synchronize()
    want = ob.asm_aggregate(ob.group_rows(q, G), ob.group_rows(a, G), ob.group_rows(lse, G), ob.group_rows(idx, G), K)
    check_aggregate((host(qbar), host(abar.float()), host(lz), host(cnt)), want)
