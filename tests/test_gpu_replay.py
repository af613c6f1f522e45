"""A dumped decode step, reloaded and replayed through the library, gives what the oracle gives on
the dumped files and what the original cache gave when it ran the same step: eviction victims,
the cache after the step (bit for bit) and the attention state, on a flat cache at its budget and
on a paged cache with a block removal after the attention."""
import numpy as np
import pytest
import torch

from memory_bounded_kv_b200 import state
from memory_bounded_kv_b200.cache import BoundedKVCache, PagedKVCache
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from oracle import paged as opaged
from gpu_util import dev, host, assert_state_close

pytestmark = pytest.mark.gpu


def test_flat_step_replays_like_the_stream_and_the_oracle(oracle, tmp_path):
    """Three sequences at the budget (M = 200 of cap 256, several tiles, a ragged last one) and
    one below it; the step evicts in three rows and appends in one, splits of 64 slots."""
    B, Hq, Hkv, d, cap, M = 4, 16, 4, 128, 256, 200
    g = rng(71)
    lens = np.array([M, M, M, 131], np.int32)
    k = normal_bf16(g, (B, Hkv, cap, d))
    v = normal_bf16(g, (B, Hkv, cap, d))
    lb = log_beta(g, (B, Hkv, cap))
    pos = np.zeros((B, Hkv, cap), np.int32)
    for b in range(B):
        for h in range(Hkv):
            pos[b, h, :lens[b]] = np.sort(g.choice(5000, lens[b], replace=False)).astype(np.int32)
    len_ = np.repeat(lens[:, None], Hkv, 1).astype(np.int32)
    c = BoundedKVCache.from_host(k, v, lb, pos, len_, Hq, M, num_splits=4, split_len=64)
    inputs = dict(q=dev(normal_bf16(g, (B, Hq, d))), k_new=dev(normal_bf16(g, (B, Hkv, d))),
                  v_new=dev(normal_bf16(g, (B, Hkv, d))), log_beta_new=dev(log_beta(g, (B, Hkv))),
                  t=dev(np.full(B, 5000, np.int32)))
    path = str(tmp_path / "flat")
    state.dump_step(path, c, inputs)

    # the original cache runs the step
    o_ref_dev, lse_ref_dev = state.replay_step(c, inputs)
    torch.cuda.synchronize()
    # the dump, reloaded, runs it again
    c2, inp2, meta = state.load_step(path)
    o2, lse2 = state.replay_step(c2, inp2)
    torch.cuda.synchronize()
    for name in ("k", "v", "log_beta", "pos", "len"):
        np.testing.assert_array_equal(host(getattr(c2, name)), host(getattr(c, name)), err_msg=name)
    np.testing.assert_array_equal(host(o2), host(o_ref_dev))
    np.testing.assert_array_equal(host(lse2), host(lse_ref_dev))

    # the oracle on the dumped files
    tens, _ = state.load(path, device="cpu")
    hc = {n: host(tens[n]).copy() for n in ("k", "v", "log_beta", "pos", "len")}
    victim = oracle.evict_insert(hc, host(tens["in_k_new"]), host(tens["in_v_new"]), host(tens["in_log_beta_new"]),
                                 host(tens["in_t"]), meta["M"])
    assert (victim[:3] >= 0).all() and (victim[3] == -1).all()
    np.testing.assert_array_equal(host(c2.victim), victim)
    for name in ("k", "v", "log_beta", "pos", "len"):
        np.testing.assert_array_equal(host(getattr(c2, name)), hc[name], err_msg=name)
    o, lse = oracle.decode_attn(host(tens["in_q"]), hc["k"], hc["v"], hc["log_beta"], hc["pos"], hc["len"],
                                host(tens["in_t"]))
    assert_state_close(host(o2), host(lse2), o, lse, "replayed step")


def test_paged_step_with_compaction_replays_like_the_oracle(oracle, tmp_path):
    """A paged cache grown over page boundaries, then one dumped step that appends, attends and
    removes a block that spans pages; the replay is compared with the oracle on the logical
    cache and the page books are checked."""
    B, Hq, Hkv, d, M = 3, 8, 2, 64, 6 * 64   # the budget is never reached
    PAGE = 64
    cache = PagedKVCache(B, Hq, Hkv, d, max_pages=6, num_pages=B * Hkv * 6, M=M, num_splits=2,
                         split_len=192, with_beta=False)
    g = rng(72)
    o = torch.zeros(B, Hq, d, device="cuda")
    lse = torch.zeros(B, Hq, device="cuda")
    steps = np.array([300, 150, 229])
    for s in range(int(steps.max())):
        t = np.where(s < steps, s, -1).astype(np.int32)
        cache.step(dev(normal_bf16(g, (B, Hq, d))), dev(normal_bf16(g, (B, Hkv, d))),
                   dev(normal_bf16(g, (B, Hkv, d))), None, dev(t), o, lse)
    torch.cuda.synchronize()
    t = steps.astype(np.int32)
    inputs = dict(q=dev(normal_bf16(g, (B, Hq, d))), k_new=dev(normal_bf16(g, (B, Hkv, d))),
                  v_new=dev(normal_bf16(g, (B, Hkv, d))), t=dev(t),
                  rm_start=dev(np.array([40, 0, 100], np.int32)), rm_len=dev(np.array([150, 0, 130], np.int32)))
    path = str(tmp_path / "paged")
    state.dump_step(path, cache, inputs)

    c2, inp2, meta = state.load_step(path)
    assert meta["kind"] == "paged"
    o2, lse2 = state.replay_step(c2, inp2)
    torch.cuda.synchronize()

    tens, _ = state.load(path, device="cpu")
    pages = dict(k=host(tens["k_pages"]), v=host(tens["v_pages"]), pos=host(tens["pos_pages"]), log_beta=None)
    hc = opaged.to_flat(pages, host(tens["table"]), host(tens["len"]), 6 * PAGE)
    hc = {n: (None if a is None else np.ascontiguousarray(a)) for n, a in hc.items()}
    oracle.evict_insert(hc, host(tens["in_k_new"]), host(tens["in_v_new"]), None, t, M)
    o_ref, lse_ref = oracle.decode_attn(host(tens["in_q"]), hc["k"], hc["v"], None, hc["pos"], hc["len"], t)
    oracle.compact_blocks(hc, host(tens["in_rm_start"]), host(tens["in_rm_len"]))
    assert_state_close(host(o2), host(lse2), o_ref, lse_ref, "replayed paged step")

    p = c2.pool
    f = opaged.to_flat(dict(k=host(p.k_pages), v=host(p.v_pages), pos=host(p.pos_pages), log_beta=None),
                       host(p.table), host(p.len), 6 * PAGE)
    np.testing.assert_array_equal(f["len"], hc["len"])
    for b in range(B):
        for h in range(Hkv):
            n = hc["len"][b, h]
            for name in ("k", "v", "pos"):
                np.testing.assert_array_equal(f[name][b, h, :n], hc[name][b, h, :n], err_msg=f"{name} b{b} h{h}")
    need = sum(-(-int(n) // PAGE) for n in hc["len"].ravel())
    assert c2.pages_in_use() == need
