"""GPU parity of kvb_decode_step (budget enforcement, insertion and attention in one launch)
against the oracle's evict_insert followed by decode_attn: victims, lengths and every cached byte
exact after each step, outputs and split states within the stated tolerances; plus records
scored for another position (the victim then comes from a scan), rows the fused step refuses (not
full) and inactive rows."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200 import _lib
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from gpu_util import dev, host, assert_state_close, assert_splits_close, GpuCache

pytestmark = pytest.mark.gpu


def full_cache(g, B, Hkv, cap, d, M, with_beta, t0):
    """Every row holds M distinct positions below t0 (shuffled over the slots)."""
    k, v = normal_bf16(g, (B, Hkv, cap, d)), normal_bf16(g, (B, Hkv, cap, d))
    lb = log_beta(g, (B, Hkv, cap)) if with_beta else None
    if with_beta:
        lb[0, 0, 5:40] = -0.125   # equal retention on a stretch: ties broken by position
    pos = np.zeros((B, Hkv, cap), np.int32)
    for b in range(B):
        for h in range(Hkv):
            pos[b, h, :M] = g.permutation(t0)[:M]
    return dict(k=k, v=v, log_beta=lb, pos=pos, len=np.full((B, Hkv), M, np.int32))


def cache_bytes_equal(gc, c, what):
    h = gc.to_host()
    np.testing.assert_array_equal(h["len"], c["len"], err_msg=what + " len")
    for key in ("k", "v", "pos") + (("log_beta",) if c["log_beta"] is not None else ()):
        np.testing.assert_array_equal(h[key], c[key], err_msg=f"{what} {key}")


@pytest.mark.parametrize("d,G,S,with_beta,M", [(128, 4, 1, True, 300), (128, 4, 5, True, 300),
                                                (64, 2, 16, True, 250), (128, 8, 3, False, 300),
                                                (64, 1, 64, True, 300)])
def test_decode_step_matches_evict_insert_then_attention(oracle, d, G, S, with_beta, M):
    """Five steps; the first attention (kvb_decode_attn) leaves the records, each kvb_decode_step
    reads one record buffer and writes the other. The oracle runs evict_insert, then
    decode_attn, on its own copy of the cache."""
    Hkv, B, cap = 2, 3, 320
    Hq = Hkv * G
    g = rng(91, d + G + S + M)
    t0 = 1000
    c = full_cache(g, B, Hkv, cap, d, M, with_beta, t0)
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    op = lp = None
    if S > 1:
        op, lp = kvb.decode_workspace(B, Hq, d, S)
    cand = [kvb.evict_candidates(B, Hkv, S), kvb.evict_candidates(B, Hkv, S)]
    victim = torch.full((B, Hkv), 7, dtype=torch.int32, device="cuda")
    o = torch.zeros(B, Hq, d, device="cuda")
    lse = torch.zeros(B, Hq, device="cuda")
    kvb.kvb_get_error()
    # the attention at t0 leaves the records for t0 + 1
    q = normal_bf16(g, (B, Hq, d))
    t = np.full(B, t0, np.int32)
    kvb.kvb_decode_attn(dev(q), gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(t), o, lse, num_splits=S,
                        o_part=op, lse_part=lp, evict_cand=cand[0])
    for step in range(1, 6):
        t = np.full(B, t0 + step, np.int32)
        q = normal_bf16(g, (B, Hq, d))
        kn, vn = normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d))
        lbn = log_beta(g, (B, Hkv)) if with_beta else None
        kvb.kvb_decode_step(dev(q), gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(t), o, lse, dev(kn), dev(vn),
                            None if lbn is None else dev(lbn), M, cand[0], cand[1], victim=victim,
                            num_splits=S, o_part=op, lse_part=lp)
        cand.reverse()
        vic_ref = oracle.evict_insert(c, kn, vn, lbn, t, M)
        o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(q, c["k"], c["v"], c["log_beta"], c["pos"], c["len"], t,
                                                          num_splits=S, want_parts=True)
        np.testing.assert_array_equal(host(victim), vic_ref, err_msg=f"step {step} victims")
        cache_bytes_equal(gc, c, f"step {step}")
        assert_state_close(host(o), host(lse), o_ref, l_ref, f"step {step}")
        if S > 1:
            assert_splits_close(host(op), host(lp), op_ref, lp_ref, f"step {step} splits")
    assert kvb.kvb_get_error() == 0


def test_decode_step_stale_records_scan_and_rows_below_budget_are_refused(oracle):
    """Records scored for another position (a skipped position) make the step find the victim by
    scanning the row's slots, as kvb_evict_insert does; a row below its budget is left unchanged
    with the empty state and KVB_DERR_STEP; an inactive row (t < 0) is empty and unchanged without
    an error. Every other row steps exactly as evict_insert + decode_attn."""
    B, Hkv, G, d, cap, M, S = 4, 2, 4, 128, 256, 256, 4
    Hq = Hkv * G
    g = rng(92, 0)
    t0 = 700
    c = full_cache(g, B, Hkv, cap, d, M, True, t0)
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    op, lp = kvb.decode_workspace(B, Hq, d, S)
    cand = [kvb.evict_candidates(B, Hkv, S), kvb.evict_candidates(B, Hkv, S)]
    o = torch.zeros(B, Hq, d, device="cuda")
    lse = torch.zeros(B, Hq, device="cuda")
    victim = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    kvb.kvb_get_error()
    # records for t0 + 1 in rows of sequences 0, 2, 3; sequence 1's records are for t0 + 2
    t_rec = np.array([t0, t0 + 1, t0, t0], np.int32)
    kvb.kvb_decode_attn(dev(normal_bf16(g, (B, Hq, d))), gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(t_rec),
                        o, lse, num_splits=S, o_part=op, lse_part=lp, evict_cand=cand[0])
    # sequence 2, kv head 1 drops below its budget
    gc.len[2, 1] = M - 1
    c["len"][2, 1] = M - 1
    before = gc.to_host()
    t = np.array([t0 + 1, t0 + 1, t0 + 1, -1], np.int32)
    q = normal_bf16(g, (B, Hq, d))
    kn, vn, lbn = normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d)), log_beta(g, (B, Hkv))
    kvb.kvb_decode_step(dev(q), gc.k, gc.v, gc.log_beta, gc.pos, gc.len, dev(t), o, lse, dev(kn), dev(vn),
                        dev(lbn), M, cand[0], cand[1], victim=victim, num_splits=S, o_part=op, lse_part=lp)
    bits = kvb.kvb_get_error()
    assert bits == _lib.DERR_STEP, bits
    after = gc.to_host()
    vic = host(victim)
    lse_h, o_h = host(lse), host(o)
    for b, h in [(2, 1), (3, 0), (3, 1)]:   # below the budget; inactive
        assert vic[b, h] == -1, (b, h)
        for key in ("k", "v", "pos", "log_beta"):
            np.testing.assert_array_equal(after[key][b, h], before[key][b, h], err_msg=f"{key} {b} {h}")
        assert np.all(lse_h[b, h * G:(h + 1) * G] == -np.inf) and not o_h[b, h * G:(h + 1) * G].any()
    # the rows that stepped, sequence 1 through the scan
    ref = {key: (None if val is None else val.copy()) for key, val in c.items()}
    vic_ref = oracle.evict_insert(ref, kn, vn, lbn, t, M)
    o_ref, l_ref = oracle.decode_attn(q, ref["k"], ref["v"], ref["log_beta"], ref["pos"], ref["len"], t)
    for b, h in [(0, 0), (0, 1), (1, 0), (1, 1), (2, 0)]:
        assert vic[b, h] == vic_ref[b, h], (b, h)
        for key in ("k", "v", "pos", "log_beta"):
            np.testing.assert_array_equal(after[key][b, h], ref[key][b, h], err_msg=f"{key} {b} {h}")
        rows = slice(h * G, (h + 1) * G)
        assert_state_close(o_h[b, rows], lse_h[b, rows], o_ref[b, rows], l_ref[b, rows], f"row {b} {h}")


def test_decode_step_host_checks():
    B, Hkv, G, d, cap, M = 1, 1, 4, 64, 64, 64
    g = rng(93, 0)
    c = full_cache(g, B, Hkv, cap, d, M, True, 200)
    gc = GpuCache(c["k"], c["v"], c["log_beta"], c["pos"], c["len"])
    q = dev(normal_bf16(g, (B, Hkv * G, d)))
    t = dev(np.array([201], np.int32))
    o = torch.zeros(B, Hkv * G, d, device="cuda")
    kn, vn = dev(normal_bf16(g, (B, Hkv, d))), dev(normal_bf16(g, (B, Hkv, d)))
    lbn = dev(log_beta(g, (B, Hkv)))
    ca, cb = kvb.evict_candidates(B, Hkv, 1), kvb.evict_candidates(B, Hkv, 1)
    args = (q, gc.k, gc.v, gc.log_beta, gc.pos, gc.len, t, o, None, kn, vn)
    with pytest.raises(ValueError):   # log_beta_new missing on a retention cache
        kvb.kvb_decode_step(*args, None, M, ca, cb)
    with pytest.raises(kvb.KvbError):   # the same record buffer in and out
        kvb.kvb_decode_step(*args, lbn, M, ca, ca)
    with pytest.raises(kvb.KvbError):   # budget above the capacity
        kvb.kvb_decode_step(*args, lbn, cap + 1, ca, cb)
