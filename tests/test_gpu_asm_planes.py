"""GPU parity of the attention-state-memory lookup over a prepared memory
(kvb_asm_prepare once, then kvb_asm_lookup_merge_planes) against the oracle: the same cases as
the lookup over fp32 centroids -- ragged K and N, exact matches and zero vectors, orderings
decided below bf16 precision, GQA-grouped tables, the assignment-only form -- plus equality of
its indices with kvb_asm_lookup_merge on the same inputs."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200.synth import normal_bf16, rng
from gpu_util import dev, host
from test_gpu_kernels import asm_inputs, check_asm, run_asm

pytestmark = pytest.mark.gpu


def run_planes(q, qbar, abar, lz, o_self, l_self, assign_only=False):
    N, H, d = q.shape
    Ht, K = qbar.shape[0], qbar.shape[1]
    planes = kvb.kvb_asm_prepare(dev(qbar))
    # tiles of 128 centroids: three bf16 parts x two K halves x 128 rows x 128 bytes
    assert planes.numel() == kvb.kvb_asm_planes_bytes(Ht, K) == Ht * (-(-K // 128)) * 3 * 2 * 128 * 128
    idx = torch.full((N, H), -7, dtype=torch.int32, device="cuda")
    o = None if assign_only else torch.zeros(N, H, d, device="cuda")
    lse = None if assign_only else torch.zeros(N, H, device="cuda")
    ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, K), dtype=torch.uint8, device="cuda")
    kvb.kvb_asm_lookup_merge_planes(dev(q), planes, Ht, K, None if assign_only else dev(abar),
                                    None if assign_only else dev(lz), None if assign_only else dev(o_self),
                                    None if assign_only else dev(l_self), idx, o, lse, ws)
    torch.cuda.synchronize()
    if assign_only:
        return host(idx)
    return host(idx), host(o), host(lse)


@pytest.mark.parametrize("N,H,K", [(1, 1, 1), (5, 3, 100), (70, 2, 700), (300, 2, 1000), (64, 4, 4096)])
def test_planes_lookup_matches_oracle(oracle, N, H, K):
    args = asm_inputs(N + K + 1, N, H, K)
    idx, o, lse = run_planes(*args)
    check_asm(oracle, *args, idx, o, lse)
    idx_lin, _, _ = run_asm(*args)
    np.testing.assert_array_equal(idx, idx_lin)   # the same fp32-exact products as the fp32 path
    assert kvb.kvb_get_error() == 0


def test_planes_exact_match_and_zero_vectors(oracle):
    N, H = 96, 2
    q, qbar, abar, lz, o_self, l_self = asm_inputs(31, N, H, N)
    for h in range(H):
        qf = (q[:, h].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qbar[h] = (qf / np.linalg.norm(qf, axis=1, keepdims=True)).astype(np.float32)
    q[5, 0] = 0
    qbar[1, 7] = 0
    idx, o, lse = run_planes(q, qbar, abar, lz, o_self, l_self)
    expect = np.tile(np.arange(N)[:, None], (1, H))
    expect[5, 0] = 0
    np.testing.assert_array_equal(idx[:, 0], expect[:, 0])
    rows = np.arange(N) != 7
    np.testing.assert_array_equal(idx[rows, 1], expect[rows, 1])
    check_asm(oracle, q, qbar, abar, lz, o_self, l_self, idx, o, lse)


@pytest.mark.parametrize("eps_exp", [9, 13, 16])
def test_planes_keep_full_fp32_centroids(oracle, eps_exp):
    """As for the fp32 path: the winner differs from the runner-up only below bf16 precision."""
    N, H, K = 3, 2, 130
    q, qbar, abar, lz, o_self, l_self = asm_inputs(40 + eps_exp, N, H, K)
    q[:] = 0
    q[:, :, 0] = 0x3F80
    qbar[:, :, 0] *= 0.1
    for h in range(H):
        qbar[h, 5] = 0
        qbar[h, 5, :2] = [1.0, 0.5]
        qbar[h, 70] = 0
        qbar[h, 70, :2] = [np.float32(1.0) + np.float32(2.0 ** -eps_exp), 0.5]
    idx, o, lse = run_planes(q, qbar, abar, lz, o_self, l_self)
    np.testing.assert_array_equal(idx, np.full((N, H), 70))
    assert check_asm(oracle, q, qbar, abar, lz, o_self, l_self, idx, o, lse) == 0


def test_planes_grouped_tables_and_assignment_only(oracle):
    import oracle.asm_build as ob
    g = rng(12, 36)
    N, H, Ht, K, d = 50, 8, 2, 300, 128
    q = normal_bf16(g, (N, H, d))
    x = g.standard_normal((Ht, K, d))
    qbar = (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)
    abar = normal_bf16(g, (Ht, K, d))
    lz = g.uniform(5, 12, (Ht, K)).astype(np.float32)
    o_self = g.standard_normal((N, H, d)).astype(np.float32)
    l_self = g.uniform(3, 9, (N, H)).astype(np.float32)
    idx, o, lse = run_planes(q, qbar, abar, lz, o_self, l_self)
    G = H // Ht
    check_asm(oracle, q, ob.expand_tables(qbar, G), ob.expand_tables(abar, G), ob.expand_tables(lz, G), o_self,
              l_self, idx, o, lse)
    np.testing.assert_array_equal(run_planes(q, qbar, abar, lz, o_self, l_self, assign_only=True), idx)


def test_planes_attention_state_memory_shape(oracle):
    """The lookup of the attention-state-memory workload (256 queries x 32 heads x 4096 entries)."""
    from memory_bounded_kv_b200 import synth
    w = synth.asm_workload()
    o_self = np.random.default_rng(3).standard_normal((w.N, w.H, w.d)).astype(np.float32)
    l_self = np.random.default_rng(4).uniform(3, 9, (w.N, w.H)).astype(np.float32)
    idx, o, lse = run_planes(w.q, w.qbar, w.abar, w.log_zbar, o_self, l_self)
    check_asm(oracle, w.q, w.qbar, w.abar, w.log_zbar, o_self, l_self, idx, o, lse)


def test_planes_more_query_blocks_than_ctas(oracle):
    """More (head, 256-query block) pairs than resident CTAs: a CTA walks two blocks, reloading the
    queries between them; a ragged last block of 32 queries and a ragged last tile of 72 centroids."""
    N, H, K = 800, 50, 200
    args = asm_inputs(77, N, H, K)
    idx, o, lse = run_planes(*args)
    check_asm(oracle, *args, idx, o, lse)
    assert kvb.kvb_get_error() == 0
