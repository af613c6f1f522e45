"""GPU parity on the five workloads, at their full sizes and in the launch
configuration the bench times (evict/insert then split-K attention with the
merge fused), against the oracle on the same seeded inputs.

1 tiny retention decode      every one of 512 steps, S = 1 and S = 4: victims, whole cache, o, lse
2 Qwen3-8B-shaped layer      victims + len every step; o, lse, whole cache at sampled steps
3 long context (131072/8192) streaming build of log beta/pos (every kv head of every sequence
                             replayed by the oracle: pos and log beta bit-exact), then 64 steps with
                             64 splits: victims every step, final and per-split states at sampled
                             steps; plain (beta = 1) variant
4 attention-state memory     all 256 x 32 indices (near-tie rule) and merged states
5 memento compaction         all 64 sequences replayed by the oracle: every compaction's lengths
                             and bytes exact; attention states on a sample
"""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200 import synth
from memory_bounded_kv_b200.cache import BoundedKVCache
from gpu_util import dev, host, assert_state_close, assert_splits_close

pytestmark = pytest.mark.gpu


def host_cache(w):
    return dict(k=w.k.copy(), v=w.v.copy(), log_beta=w.log_beta.copy(), pos=w.pos.copy(), len=w.len.copy())


def device_step(cache, inp, o, lse):
    cache.step(dev(inp["q"]), dev(inp["k_new"]), dev(inp["v_new"]), dev(inp["log_beta_new"]), dev(inp["t"]), o, lse)


def compare_cache(cache, c, what, b_max=None):
    ln = host(cache.len) if b_max is None else host(cache.len)[:b_max]
    np.testing.assert_array_equal(ln, c["len"] if b_max is None else c["len"][:b_max], err_msg=what)
    for key, t in (("k", cache.k), ("v", cache.v), ("pos", cache.pos), ("log_beta", cache.log_beta)):
        if t is None:
            continue
        h = host(t if b_max is None else t[:b_max])
        ref = c[key] if b_max is None else c[key][:b_max]
        for b in range(h.shape[0]):
            for g in range(h.shape[1]):
                n = ln[b, g]
                np.testing.assert_array_equal(h[b, g, :n], ref[b, g, :n], err_msg=f"{what} {key} b{b} g{g}")


@pytest.mark.parametrize("S", [1, 4])
def test_tiny_decode_every_step(oracle, S):
    w = synth.decode_workload(1)
    cache = BoundedKVCache.from_host(w.k, w.v, w.log_beta, w.pos, w.len, w.Hq, w.M, num_splits=S)
    c = host_cache(w)
    o = torch.zeros(w.B, w.Hq, w.d, device="cuda")
    lse = torch.zeros(w.B, w.Hq, device="cuda")
    for step in range(w.steps):
        inp = w.step_inputs(step)
        device_step(cache, inp, o, lse)
        v_ref = oracle.evict_insert(c, inp["k_new"], inp["v_new"], inp["log_beta_new"], inp["t"], w.M)
        o_ref, l_ref = oracle.decode_attn(inp["q"], c["k"], c["v"], c["log_beta"], c["pos"], c["len"], inp["t"])
        np.testing.assert_array_equal(host(cache.victim), v_ref, err_msg=f"step {step}")
        assert_state_close(host(o), host(lse), o_ref, l_ref, f"step {step}")
        if step % 64 == 0 or step == w.steps - 1:
            compare_cache(cache, c, f"step {step}")


def test_qwen3_layer_sampled_steps(oracle):
    w = synth.decode_workload(2)
    S = w.splits[0]
    cache = BoundedKVCache.from_host(w.k, w.v, w.log_beta, w.pos, w.len, w.Hq, w.M, num_splits=S)
    c = host_cache(w)
    o = torch.zeros(w.B, w.Hq, w.d, device="cuda")
    lse = torch.zeros(w.B, w.Hq, device="cuda")
    sampled = {0, 1, 2, 255, 511, 1023}
    for step in range(w.steps):
        inp = w.step_inputs(step)
        device_step(cache, inp, o, lse)
        v_ref = oracle.evict_insert(c, inp["k_new"], inp["v_new"], inp["log_beta_new"], inp["t"], w.M)
        np.testing.assert_array_equal(host(cache.victim), v_ref, err_msg=f"step {step}")
        if step in sampled:
            o_ref, l_ref = oracle.decode_attn(inp["q"], c["k"], c["v"], c["log_beta"], c["pos"], c["len"], inp["t"])
            assert_state_close(host(o), host(lse), o_ref, l_ref, f"step {step}")
            compare_cache(cache, c, f"step {step}")


def long_context_build(w, cache):
    """Stream positions cap .. 131071 through budget enforcement (log beta and pos only)."""
    blocks = (synth.CONFIG3_LOGICAL_T - w.cap) // synth.STREAM_BLOCK
    for blk in range(blocks):
        lbs = dev(synth.stream_log_beta(w, blk))
        base = w.cap + blk * synth.STREAM_BLOCK
        ts = dev(np.repeat((base + np.arange(synth.STREAM_BLOCK, dtype=np.int32))[:, None], w.B, axis=1))
        for i in range(synth.STREAM_BLOCK):
            kvb.kvb_evict_insert(cache.k, cache.v, cache.log_beta, cache.pos, cache.len, None, None, lbs[i], ts[i],
                                 w.M)
    return blocks


def test_long_context_stream_and_decode(oracle):
    w = synth.decode_workload(3)
    S = w.splits[0]
    cache = BoundedKVCache.from_host(w.k, w.v, w.log_beta, w.pos, w.len, w.Hq, w.M, num_splits=S)
    blocks = long_context_build(w, cache)
    torch.cuda.synchronize()
    # the oracle replays the stream for every (sequence, kv head), the heads spread over the host's
    # cores by its parallel driver (the serial functions on each head's slice)
    sub = dict(k=np.zeros((w.B, w.Hkv, w.cap, 8), np.uint16), v=np.zeros((w.B, w.Hkv, w.cap, 8), np.uint16),
               log_beta=w.log_beta.copy(), pos=w.pos.copy(), len=np.full((w.B, w.Hkv), w.cap, np.int32))
    for blk in range(blocks):
        lbs = synth.stream_log_beta(w, blk)
        base = w.cap + blk * synth.STREAM_BLOCK
        ts = np.repeat((base + np.arange(synth.STREAM_BLOCK, dtype=np.int32))[:, None], w.B, axis=1)
        oracle.decode_steps_threads(sub, None, None, None, lbs, ts, w.M)
    gpos, glb = host(cache.pos), host(cache.log_beta)
    np.testing.assert_array_equal(host(cache.len), sub["len"])
    np.testing.assert_array_equal(gpos, sub["pos"])
    np.testing.assert_array_equal(glb, sub["log_beta"])
    # and the invariants: every head full, unique positions below the logical length
    assert np.all(host(cache.len) == w.M)
    assert np.all(gpos < synth.CONFIG3_LOGICAL_T) and all(
        len(np.unique(gpos[b, g])) == w.M for b in range(w.B) for g in range(w.Hkv))
    # survivors get their K/V, then 64 decode steps with 64 splits
    k, v = synth.long_context_kv(w)
    cache.k.copy_(dev(k))
    cache.v.copy_(dev(v))
    c = dict(k=k, v=v, log_beta=glb.copy(), pos=gpos.copy(), len=host(cache.len))
    o = torch.zeros(w.B, w.Hq, w.d, device="cuda")
    lse = torch.zeros(w.B, w.Hq, device="cuda")
    o_plain = torch.zeros_like(o)
    lse_plain = torch.zeros_like(lse)
    for step in range(w.steps):
        inp = w.step_inputs(step)
        device_step(cache, inp, o, lse)
        v_ref = oracle.evict_insert(c, inp["k_new"], inp["v_new"], inp["log_beta_new"], inp["t"], w.M)
        np.testing.assert_array_equal(host(cache.victim), v_ref, err_msg=f"step {step}")
        if step in (0, 1, 31, 63):
            o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(inp["q"], c["k"], c["v"], c["log_beta"], c["pos"],
                                                              c["len"], inp["t"], num_splits=S, want_parts=True)
            assert_state_close(host(o), host(lse), o_ref, l_ref, f"step {step}")
            assert_splits_close(host(cache.o_part), host(cache.lse_part), op_ref, lp_ref, f"step {step} splits")
            # plain variant: beta = 1 (no log beta, no positions read)
            cache.attend(dev(inp["q"]), None, o_plain, lse_plain, use_beta=False)
            o_ref, l_ref = oracle.decode_attn(inp["q"], c["k"], c["v"], None, c["pos"], c["len"], None)
            assert_state_close(host(o_plain), host(lse_plain), o_ref, l_ref, f"plain step {step}")


def test_memory_lookup_workload_full(oracle):
    w = synth.asm_workload()
    N, H, Hkv, d = w.N, w.H, w.Hkv, w.d
    # self attention of each query over its causal prefix of the shared cache (batch stride 0)
    kd = dev(w.k).expand(N, Hkv, w.L, d)
    vd = dev(w.v).expand(N, Hkv, w.L, d)
    posd = dev(w.pos).expand(N, Hkv, w.L)
    o_self = torch.zeros(N, H, d, device="cuda")
    l_self = torch.zeros(N, H, device="cuda")
    op, lp = kvb.decode_workspace(N, H, d, 4)
    kvb.kvb_decode_attn(dev(w.q), kd, vd, None, posd, dev(w.len), dev(w.t), o_self, l_self, num_splits=4,
                        split_len=512, o_part=op, lse_part=lp)
    os_ref, ls_ref = oracle.decode_attn(w.q, w.k, w.v, None, w.pos, w.len, w.t, kv_batch_stride=0,
                                        meta_batch_stride=0)
    assert_state_close(host(o_self), host(l_self), os_ref, ls_ref, "self attention")
    idx = torch.zeros(N, H, dtype=torch.int32, device="cuda")
    o = torch.zeros(N, H, d, device="cuda")
    lse = torch.zeros(N, H, device="cuda")
    ws = torch.empty(kvb.kvb_asm_workspace_bytes(N, H, w.K), dtype=torch.uint8, device="cuda")
    kvb.kvb_asm_lookup_merge(dev(w.q), dev(w.qbar), dev(w.abar), dev(w.log_zbar), o_self, l_self, idx, o, lse, ws)
    # the oracle merges the same float32 self state the GPU merged
    from test_gpu_kernels import check_asm
    check_asm(oracle, w.q, w.qbar, w.abar, w.log_zbar, host(o_self), host(l_self), host(idx), host(o), host(lse))


def test_memento_compaction_workload(oracle):
    """Scope: the oracle replays every one of the 64 sequences (append at every step, removal at
    every memento end). At every compaction step the lengths of all 64 sequences are compared,
    and the K, V and pos bytes of every sequence compacted at that step, over its whole length;
    the whole batch's bytes at eight spread compaction steps and at the end. Attention states
    are compared on a sample: sequences 0, 1, 31, 63 around their compactions and at 20 random
    steps, plus every sequence at 4 of those steps."""
    w = synth.memento_workload()
    SPLIT_LEN = 512
    S = -(-w.cap // SPLIT_LEN)
    cache = BoundedKVCache(w.B, w.Hq, w.Hkv, w.d, w.cap, w.cap, num_splits=S, split_len=SPLIT_LEN, with_beta=False)
    c = dict(k=np.zeros((w.B, w.Hkv, w.cap, w.d), np.uint16), v=np.zeros((w.B, w.Hkv, w.cap, w.d), np.uint16),
             log_beta=None, pos=np.zeros((w.B, w.Hkv, w.cap), np.int32), len=np.zeros((w.B, w.Hkv), np.int32))
    o = torch.zeros(w.B, w.Hq, w.d, device="cuda")
    lse = torch.zeros(w.B, w.Hq, device="cuda")
    ends = np.cumsum(w.blk + w.mem, axis=1) - 1
    watch = [0, 1, 31, 63]
    check_steps = set()
    for b in watch:
        for e in ends[b]:
            check_steps.update({int(e) - 1, int(e), int(e) + 1})
    rand_steps = np.random.default_rng(5).integers(0, w.steps, 20).tolist()
    check_steps.update(rand_steps)
    full_attn_steps = set(rand_steps[:4])
    comp_list = w.compaction_steps().tolist()
    comp_steps = set(comp_list)
    full_cache_steps = set(comp_list[:: max(1, len(comp_list) // 8)])
    pool = [w.step_inputs(s) for s in range(w.pool)]
    pool_dev = [{key: dev(val) for key, val in inp.items() if key != "t"} for inp in pool]

    def compare_seq(b, what):
        n = int(c["len"][b].max())
        for key, t in (("k", cache.k), ("v", cache.v), ("pos", cache.pos)):
            h = host(t[b, :, :n])
            for g in range(w.Hkv):
                m = c["len"][b, g]
                np.testing.assert_array_equal(h[g, :m], c[key][b, g, :m], err_msg=f"{what} {key} b{b} g{g}")

    n_checked = n_compared = 0
    for step in range(w.steps):
        inp = pool[step % w.pool]
        t = np.where(step < w.total, step, -1).astype(np.int32)
        td = dev(t)
        pd = pool_dev[step % w.pool]
        cache.insert(pd["k_new"], pd["v_new"], None, td)
        cache.attend(pd["q"], td, o, lse)
        oracle.evict_insert(c, inp["k_new"], inp["v_new"], None, t, w.cap)
        if step in check_steps:
            sel = slice(None) if step in full_attn_steps else watch   # a slice: no copy of the whole cache
            o_ref, l_ref = oracle.decode_attn(inp["q"][sel], c["k"][sel], c["v"][sel], None, c["pos"][sel],
                                              c["len"][sel], t[sel])
            assert_state_close(host(o[sel]), host(lse[sel]), o_ref, l_ref, f"step {step}")
            n_checked += 1
        if step in comp_steps:
            rs, rl = w.compaction(step)
            cache.compact(dev(rs), dev(rl))
            oracle.compact_blocks(c, rs, rl)
            np.testing.assert_array_equal(host(cache.len), c["len"], err_msg=f"len after compaction at {step}")
            for b in np.nonzero(rl)[0]:
                compare_seq(int(b), f"compaction at {step}")
                n_compared += 1
            if step in full_cache_steps:
                for b in range(w.B):
                    compare_seq(b, f"whole batch at {step}")
    assert n_checked >= 40
    assert n_compared == int((w.blk > 0).sum())   # every block removal was compared
    for b in range(w.B):
        compare_seq(b, "end")
    # finished sequences hold exactly their mementos
    np.testing.assert_array_equal(host(cache.len)[:, 0], w.mem.sum(axis=1))
