"""GPU parity of kvb_evict_insert, kvb_compact_blocks, kvb_merge_states and
kvb_asm_lookup_merge against the oracle on small seeded inputs.
Indices, victims, lengths and cache bytes are compared bit for bit."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from memory_bounded_kv_b200 import _lib
from gpu_util import dev, host, GpuCache, assert_state_close

pytestmark = pytest.mark.gpu


def empty_cache(B, Hkv, cap, d, with_beta=True):
    return dict(k=np.zeros((B, Hkv, cap, d), np.uint16), v=np.zeros((B, Hkv, cap, d), np.uint16),
                log_beta=np.zeros((B, Hkv, cap), np.float32) if with_beta else None,
                pos=np.zeros((B, Hkv, cap), np.int32), len=np.zeros((B, Hkv), np.int32))


def assert_cache_equal(gc: GpuCache, c: dict, what=""):
    h = gc.to_host()
    np.testing.assert_array_equal(h["len"], c["len"], err_msg=what + " len")
    for b in range(c["len"].shape[0]):
        for g in range(c["len"].shape[1]):
            n = c["len"][b, g]
            for key in ("k", "v", "pos") + (("log_beta",) if c["log_beta"] is not None else ()):
                np.testing.assert_array_equal(h[key][b, g, :n], c[key][b, g, :n], err_msg=f"{what} {key} {b} {g}")


@pytest.mark.parametrize("mode", ["random", "const", "null", "meta_only", "ties"])
def test_evict_insert_stream_bit_exact(oracle, mode):
    B, Hkv, cap, d, M = 3, 4, 96, 128, 80
    c = empty_cache(B, Hkv, cap, d, with_beta=(mode != "null"))
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    victim = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    for t in range(300):
        g = rng(20, t)
        kn, vn = normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d))
        lb = log_beta(g, (B, Hkv))
        if mode == "const":
            lb[:] = -0.25
        if mode == "ties":   # few distinct values: many equal scores
            lb = (-0.125 * g.integers(0, 4, (B, Hkv))).astype(np.float32)
        tt = np.full(B, t, np.int32)
        if t % 17 == 5:
            tt[1] = -1       # an inactive sequence this step
        if mode == "meta_only":
            kn = vn = None
        lbn = None if mode == "null" else lb
        v_ref = oracle.evict_insert(c, kn, vn, lbn, tt, M)
        kvb.kvb_evict_insert(gc.k, gc.v, gc.log_beta, gc.pos, gc.len, None if kn is None else dev(kn),
                             None if vn is None else dev(vn), None if lbn is None else dev(lbn), dev(tt), M, victim)
        np.testing.assert_array_equal(host(victim), v_ref, err_msg=f"victim at t={t}")
        if t % 23 == 0 or t == 299:
            assert_cache_equal(gc, c, f"t={t}")


def test_evict_insert_large_cache_bit_exact(oracle):
    """Full-budget eviction over 4096 slots (the size of the Qwen3-8B-shaped workload)."""
    B, Hkv, cap, d, M = 2, 8, 4096, 128, 4096
    g = rng(21, 0)
    c = dict(k=normal_bf16(g, (B, Hkv, cap, d)), v=normal_bf16(g, (B, Hkv, cap, d)),
             log_beta=log_beta(g, (B, Hkv, cap)), pos=np.tile(np.arange(cap, dtype=np.int32), (B, Hkv, 1)),
             len=np.full((B, Hkv), cap, np.int32))
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    victim = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    for t in range(cap, cap + 40):
        g = rng(21, t)
        kn, vn, lb = normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d)), log_beta(g, (B, Hkv))
        tt = np.full(B, t, np.int32)
        v_ref = oracle.evict_insert(c, kn, vn, lb, tt, M)
        kvb.kvb_evict_insert(gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(kn), dev(vn), dev(lb), dev(tt), M, victim)
        np.testing.assert_array_equal(host(victim), v_ref)
    assert_cache_equal(gc, c)


@pytest.mark.parametrize("S,with_beta", [(1, True), (3, True), (16, True), (5, False)])
def test_attention_leaves_exact_eviction_candidates(oracle, S, with_beta):
    """Each split's record is the slot the oracle evicts at t + 1 among that split's slots."""
    B, Hq, Hkv, d, cap = 2, 8, 2, 128, 300
    g = rng(25, S)
    q = normal_bf16(g, (B, Hq, d))
    k, v = normal_bf16(g, (B, Hkv, cap, d)), normal_bf16(g, (B, Hkv, cap, d))
    lb = log_beta(g, (B, Hkv, cap)) if with_beta else None
    if with_beta:
        lb[0, 0, 10:20] = -0.125   # equal scores for equal distances: ties resolved by position
    pos = np.stack([np.stack([g.permutation(2 * cap)[:cap] for _ in range(Hkv)]) for _ in range(B)]).astype(np.int32)
    ln = np.array([[300, 257], [1, 64]], np.int32)
    t = np.full(B, 2 * cap + 1, np.int32)
    o = torch.zeros(B, Hq, d, device="cuda")
    op, lp = kvb.decode_workspace(B, Hq, d, S)
    cand = kvb.evict_candidates(B, Hkv, S)
    kvb.kvb_decode_attn(dev(q), dev(k), dev(v), None if lb is None else dev(lb), dev(pos), dev(ln), dev(t), o,
                        num_splits=S, o_part=op, lse_part=lp, evict_cand=cand)
    rec = host(cand).reshape(B, Hkv, S, 2)
    slots = (rec[..., 1] & 0xffffffff).astype(np.int64)
    slots = np.where(slots >= 2**31, slots - 2**32, slots)
    # every record carries the position it was scored for
    stamps = (rec[..., 1] >> 32).astype(np.int64)
    assert np.all(stamps == (t + 1)[:, None, None])
    for b in range(B):
        for gg in range(Hkv):
            n = ln[b, gg]
            C = -(-n // S)
            for j in range(S):
                s0, s1 = min(j * C, n), min((j + 1) * C, n)
                if s1 <= s0:
                    assert slots[b, gg, j] == -1
                    continue
                sub = dict(k=np.zeros((1, 1, s1 - s0, 8), np.uint16), v=np.zeros((1, 1, s1 - s0, 8), np.uint16),
                           log_beta=None if lb is None else lb[b, gg, s0:s1][None, None].copy(),
                           pos=pos[b, gg, s0:s1][None, None].copy(), len=np.array([[s1 - s0]], np.int32))
                vic = oracle.evict_insert(sub, None, None, None if lb is None else np.zeros((1, 1), np.float32),
                                          np.array([t[b] + 1], np.int32), s1 - s0)
                assert slots[b, gg, j] == s0 + vic[0, 0], (b, gg, j)


def _crossing_cache(M, T0):
    """A full cache whose victim at T0 + 1 is slot 3 and at T0 + 2 is slot 7: slot 3 (pos T0 - 10,
    log beta -0.2) scores (T - pos) log beta = -2.2 then -2.4, slot 7 (pos T0 - 1, log beta -1)
    -2.0 then -3.0; every other slot keeps log beta -1e-4."""
    Hkv, d = 1, 64
    g = rng(31, 0)
    k, v = normal_bf16(g, (1, Hkv, M, d)), normal_bf16(g, (1, Hkv, M, d))
    lb = np.full((1, Hkv, M), -1e-4, np.float32)
    pos = np.arange(T0 - 2 * M, T0 - M, dtype=np.int32).reshape(1, 1, M).copy()
    lb[0, 0, 3], pos[0, 0, 3] = -0.2, T0 - 10
    lb[0, 0, 7], pos[0, 0, 7] = -1.0, T0 - 1
    return dict(k=k, v=v, log_beta=lb, pos=pos, len=np.full((1, Hkv), M, np.int32))


@pytest.mark.parametrize("skip", [1, 2])
def test_evict_candidates_only_for_the_position_they_were_scored_for(oracle, skip):
    """Attention at T0 leaves candidates for T0 + 1. Inserting at T0 + 1 uses them; inserting at
    T0 + 2 (a skipped position) must not: the ranking changed, and the victim is the scan's."""
    M, T0, S = 64, 1000, 4
    c = _crossing_cache(M, T0)
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    g = rng(32, skip)
    q = normal_bf16(g, (1, 4, 64))
    o = torch.zeros(1, 4, 64, device="cuda")
    op, lp = kvb.decode_workspace(1, 4, 64, S)
    cand = kvb.evict_candidates(1, 1, S)
    kvb.kvb_decode_attn(dev(q), gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(np.array([T0], np.int32)), o,
                        num_splits=S, o_part=op, lse_part=lp, evict_cand=cand)
    kn, vn, lbn = normal_bf16(g, (1, 1, 64)), normal_bf16(g, (1, 1, 64)), np.full((1, 1), -0.5, np.float32)
    t_ins = np.array([T0 + skip], np.int32)
    victim = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    kvb.kvb_evict_insert(gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(kn), dev(vn), dev(lbn), dev(t_ins), M,
                         victim, cand=cand, cand_n=S)
    want = oracle.evict_insert(c, kn, vn, lbn, t_ins, M)
    assert int(want[0, 0]) == (3 if skip == 1 else 7)
    np.testing.assert_array_equal(host(victim), want)
    assert_cache_equal(gc, c)
    assert kvb.kvb_get_error() == 0


@pytest.mark.parametrize("S", [1, 3])
def test_bounded_wait_runs_out_and_leaves_the_empty_state(oracle, S):
    """The testing hook makes every producer withhold its copies, so each CTA's first bounded
    wait on a tile runs out (after 20 us). The call returns, the device error word reports
    KVB_DERR_TIMEOUT, every row is the empty state, the candidates name no slot, and the next
    call on the same context is correct again."""
    B, Hq, Hkv, d, cap = 2, 8, 2, 128, 200
    g = rng(33, S)
    q, k, v = normal_bf16(g, (B, Hq, d)), normal_bf16(g, (B, Hkv, cap, d)), normal_bf16(g, (B, Hkv, cap, d))
    lb = log_beta(g, (B, Hkv, cap))
    pos = np.tile(np.arange(cap, dtype=np.int32), (B, Hkv, 1))
    ln = np.array([[200, 130], [77, 1]], np.int32)
    t = np.full(B, cap + 2, np.int32)
    args = [dev(x) for x in (q, k, v, lb, pos, ln, t)]
    op = lp = None
    if S > 1:
        op, lp = kvb.decode_workspace(B, Hq, d, S)
    cand = kvb.evict_candidates(B, Hkv, S)
    kvb.kvb_get_error()
    o = torch.full((B, Hq, d), 7.0, device="cuda")
    lse = torch.full((B, Hq), 7.0, device="cuda")
    kvb.kvb_test_withhold_next_decode(20_000)
    kvb.kvb_decode_attn(*args, o, lse, num_splits=S, o_part=op, lse_part=lp, evict_cand=cand)
    bits = kvb.kvb_get_error()
    assert bits & _lib.DERR_TIMEOUT, bits
    assert np.all(host(lse) == -np.inf) and not host(o).any()
    rec = host(cand).reshape(B, Hkv, S, 2)
    assert np.all((rec[..., 1] & 0xffffffff) == 0xffffffff)   # slot -1 everywhere
    # the hook armed one launch only: the same call now matches the oracle
    kvb.kvb_decode_attn(*args, o, lse, num_splits=S, o_part=op, lse_part=lp, evict_cand=cand)
    assert kvb.kvb_get_error() == 0
    o_ref, l_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    assert_state_close(host(o), host(lse), o_ref, l_ref, "after the timeout")


def test_evict_insert_bad_length_flags_error():
    c = empty_cache(1, 2, 8, 64)
    c["len"][0, 1] = 9
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    g = rng(22, 0)
    kvb.kvb_get_error()
    kvb.kvb_evict_insert(gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(normal_bf16(g, (1, 2, 64))),
                         dev(normal_bf16(g, (1, 2, 64))), dev(log_beta(g, (1, 2))), dev(np.array([0], np.int32)), 8)
    assert kvb.kvb_get_error() & 1
    assert host(gc.len).tolist() == [[1, 9]]


@pytest.mark.parametrize("d", [64, 128])
def test_compact_blocks_bit_exact(oracle, d):
    B, Hkv, cap = 6, 2, 700
    g = rng(23, d)
    c = dict(k=normal_bf16(g, (B, Hkv, cap, d)), v=normal_bf16(g, (B, Hkv, cap, d)),
             log_beta=log_beta(g, (B, Hkv, cap)), pos=np.tile(np.arange(cap, dtype=np.int32), (B, Hkv, 1)),
             len=np.array([[700, 650]] * B, np.int32))
    # no-op, overlap (tail > removed), no overlap, remove all, remove the tail, a single slot
    rs = np.array([0, 10, 5, 0, 600, 300], np.int32)
    rl = np.array([0, 3, 500, 650, 50, 1], np.int32)
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    oracle.compact_blocks(c, rs, rl)
    kvb.kvb_compact_blocks(gc.k, gc.v, gc.pos, gc.log_beta, gc.len, dev(rs), dev(rl))
    assert_cache_equal(gc, c)


def test_compact_blocks_invalid_range_flags_error_and_leaves_head():
    B, Hkv, cap, d = 1, 2, 64, 64
    g = rng(24, 0)
    c = dict(k=normal_bf16(g, (B, Hkv, cap, d)), v=normal_bf16(g, (B, Hkv, cap, d)), log_beta=None,
             pos=np.tile(np.arange(cap, dtype=np.int32), (B, Hkv, 1)), len=np.array([[64, 20]], np.int32))
    gc = GpuCache(c["k"], c["v"], None, c["pos"], c["len"])
    kvb.kvb_get_error()
    kvb.kvb_compact_blocks(gc.k, gc.v, gc.pos, None, gc.len, dev(np.array([10], np.int32)),
                           dev(np.array([15], np.int32)))
    assert kvb.kvb_get_error() & 4
    h = gc.to_host()
    assert h["len"].tolist() == [[49, 20]]
    np.testing.assert_array_equal(h["k"][0, 1], c["k"][0, 1])


@pytest.mark.parametrize("n,R,d", [(1, 5, 128), (2, 7, 128), (64, 128, 128), (5, 3, 33), (17, 40, 64)])
def test_merge_states(oracle, n, R, d):
    g = np.random.default_rng(n * 100 + d)
    o_in = g.standard_normal((n, R, d)).astype(np.float32)
    lse_in = g.uniform(-20, 20, (n, R)).astype(np.float32)
    lse_in[g.random((n, R)) < 0.2] = -np.inf   # empty states
    lse_in[:, 0] = -np.inf                     # an all-empty row
    o_out = torch.zeros(R, d, device="cuda")
    lse_out = torch.zeros(R, device="cuda")
    kvb.kvb_merge_states(dev(o_in), dev(lse_in), o_out, lse_out)
    o_ref, l_ref = oracle.merge_states(o_in.astype(np.float64), lse_in.astype(np.float64))
    assert_state_close(host(o_out), host(lse_out), o_ref, l_ref)


def test_merge_states_strided_split_layout(oracle):
    """States laid out as kvb_decode_attn's o_part [R, S, d] (state index inside the row)."""
    R, S, d = 64, 9, 128
    g = np.random.default_rng(5)
    op = g.standard_normal((R, S, d)).astype(np.float32)
    lp = g.uniform(-5, 5, (R, S)).astype(np.float32)
    opd, lpd = dev(op), dev(lp)
    o_out = torch.zeros(R, d, device="cuda")
    lse_out = torch.zeros(R, device="cuda")
    kvb.kvb_merge_states(opd.transpose(0, 1), lpd.transpose(0, 1), o_out, lse_out)
    o_ref, l_ref = oracle.merge_states(op.transpose(1, 0, 2).astype(np.float64), lp.T.astype(np.float64))
    assert_state_close(host(o_out), host(lse_out), o_ref, l_ref)


def asm_inputs(seed, N, H, K, d=128, unit=True):
    g = rng(seed, 3)
    x = g.standard_normal((H, K, d))
    qbar = (x / np.linalg.norm(x, axis=-1, keepdims=True) if unit else x).astype(np.float32)
    abar = normal_bf16(g, (H, K, d))
    lz = g.uniform(5, 12, (H, K)).astype(np.float32)
    q = normal_bf16(g, (N, H, d))
    o_self = g.standard_normal((N, H, d)).astype(np.float32)
    l_self = g.uniform(3, 9, (N, H)).astype(np.float32)
    return q, qbar, abar, lz, o_self, l_self


def run_asm(q, qbar, abar, lz, o_self, l_self):
    N, H, d = q.shape
    K = qbar.shape[1]
    idx = torch.zeros(N, H, dtype=torch.int32, device="cuda")
    o = torch.zeros(N, H, d, device="cuda")
    lse = torch.zeros(N, H, device="cuda")
    ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, K), dtype=torch.uint8, device="cuda")
    kvb.kvb_asm_lookup_merge(dev(q), dev(qbar), dev(abar), dev(lz), dev(o_self), dev(l_self), idx, o, lse, ws)
    return host(idx), host(o), host(lse)


def check_asm(oracle, q, qbar, abar, lz, o_self, l_self, idx, o, lse):
    """Indices: equal to the oracle's, or a near tie (oracle cosines within 1e-6);
    merged state: against the oracle's merge with the GPU's index."""
    idx_ref, o_ref, l_ref = oracle.asm_lookup_merge(q, qbar, abar, lz, o_self, l_self)
    diff = np.argwhere(idx != idx_ref)
    for n, h in diff:
        cos = oracle.asm_cosines(q, qbar, n, h)
        assert abs(cos[idx[n, h]] - cos[idx_ref[n, h]]) <= 1e-6, (n, h, idx[n, h], idx_ref[n, h])
    if len(diff):
        # recompute the reference merge with the GPU's (near-tie) choices
        idx_ref = idx
        N, H, d = q.shape
        for n, h in diff:
            k = idx[n, h]
            one = oracle.asm_lookup_merge(q[n:n + 1, h:h + 1], qbar[h:h + 1, k:k + 1], abar[h:h + 1, k:k + 1],
                                          lz[h:h + 1, k:k + 1], o_self[n:n + 1, h:h + 1], l_self[n:n + 1, h:h + 1])
            o_ref[n, h], l_ref[n, h] = one[1][0, 0], one[2][0, 0]
    assert_state_close(o, lse, o_ref, l_ref, "asm merge")
    return len(diff)


@pytest.mark.parametrize("N,H,K", [(1, 1, 1), (5, 3, 100), (70, 2, 700), (64, 4, 4096)])
def test_asm_lookup_merge(oracle, N, H, K):
    args = asm_inputs(N + K, N, H, K)
    idx, o, lse = run_asm(*args)
    check_asm(oracle, *args, idx, o, lse)


def test_asm_exact_match_and_zero_vectors(oracle):
    N, H, d = 96, 2, 128
    q, qbar, abar, lz, o_self, l_self = asm_inputs(31, N, H, N)
    for h in range(H):   # centroid k is query k itself: unique maximum cos = 1 at k
        qf = (q[:, h].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qbar[h] = (qf / np.linalg.norm(qf, axis=1, keepdims=True)).astype(np.float32)
    q[5, 0] = 0          # zero query: every cosine is 0 -> index 0
    qbar[1, 7] = 0       # zero centroid: cosine 0
    idx, o, lse = run_asm(q, qbar, abar, lz, o_self, l_self)
    expect = np.tile(np.arange(N)[:, None], (1, H))
    expect[5, 0] = 0
    np.testing.assert_array_equal(idx[:, 0], expect[:, 0])
    rows = np.arange(N) != 7   # centroid 7 of head 1 is the zero vector: cos 0, not the maximum
    np.testing.assert_array_equal(idx[rows, 1], expect[rows, 1])
    check_asm(oracle, q, qbar, abar, lz, o_self, l_self, idx, o, lse)


@pytest.mark.parametrize("eps_exp", [9, 13, 16])
def test_asm_lookup_uses_full_fp32_centroids(oracle, eps_exp):
    """Centroids whose order is decided below bf16 precision. For q = e0, centroid
    (c0, 0.5, 0, ...) has cos c0 / sqrt(c0^2 + 0.25), increasing in c0; c0 = 1 + 2^-e
    beats c0 = 1 by about 0.18 * 2^-e, far above the near-tie tolerance, yet 1 + 2^-e
    rounds to 1 in bf16 (e >= 9). The winner sits at the higher index, so a contraction
    that loses the low bits of the centroid ties and picks the lower one."""
    N, H, K, d = 3, 2, 130, 128
    q, qbar, abar, lz, o_self, l_self = asm_inputs(40 + eps_exp, N, H, K)
    q[:] = 0
    q[:, :, 0] = 0x3F80                                    # bf16 1.0: q = e0 in every row and head
    qbar[:, :, 0] *= 0.1                                   # fillers: cos <= 0.1
    for h in range(H):
        qbar[h, 5] = 0
        qbar[h, 5, :2] = [1.0, 0.5]
        qbar[h, 70] = 0
        qbar[h, 70, :2] = [np.float32(1.0) + np.float32(2.0 ** -eps_exp), 0.5]
    assert np.float32(qbar[0, 70, 0]) != np.float32(1.0)
    idx, o, lse = run_asm(q, qbar, abar, lz, o_self, l_self)
    np.testing.assert_array_equal(idx, np.full((N, H), 70))
    assert check_asm(oracle, q, qbar, abar, lz, o_self, l_self, idx, o, lse) == 0
