"""GPU parity of the paged cache (kvb_paged_*) against the flat oracle on the logical cache.

Each paged operation computes its flat counterpart on the logical cache (oracle/paged.py maps
pages to the flat layout): budget enforcement + insertion (appends across page boundaries,
evictions with and without the attention's candidates), attention over pages (splits of whole
pages, bias, candidates for the next position), and in-place block removal (tails longer than
the range, the range at the end, everything removed). Victims, lengths and every byte of the
logical cache are compared exactly; attention states within the tolerances of gpu_util. The
page bookkeeping is checked too: pages in use = the pages the lengths need, each used once,
the rest on the free stack."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200 import _lib, synth
from memory_bounded_kv_b200.cache import PagedKVCache
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from oracle import paged as opaged
from gpu_util import dev, host, assert_state_close, assert_splits_close

pytestmark = pytest.mark.gpu
PAGE = _lib.PAGE_SLOTS


def logical(pool, cap=None):
    pages = dict(k=host(pool.k_pages), v=host(pool.v_pages), pos=host(pool.pos_pages),
                 log_beta=None if pool.log_beta_pages is None else host(pool.log_beta_pages))
    return opaged.to_flat(pages, host(pool.table), host(pool.len), cap)


def check_books(pool):
    """Pages in use are exactly the pages the lengths need, each once; the others are free."""
    ln, table = host(pool.len), host(pool.table)
    fc = int(host(pool.free_count)[0])
    need = 0
    used = []
    for b in range(pool.B):
        for g in range(pool.Hkv):
            k = -(-int(ln[b, g]) // PAGE)
            need += k
            assert np.all(table[b, g, :k] >= 0) and np.all(table[b, g, k:] == -1), (b, g)
            used += table[b, g, :k].tolist()
    free = host(pool.free_pages)[:fc].tolist()
    assert fc == pool.num_pages - need
    assert sorted(used + free) == list(range(pool.num_pages))


def compare(cache, c, what):
    f = logical(cache.pool, c["k"].shape[2])
    np.testing.assert_array_equal(f["len"], c["len"], err_msg=what)
    for key in ("k", "v", "pos", "log_beta"):
        if c.get(key) is None:
            continue
        for b in range(c["len"].shape[0]):
            for g in range(c["len"].shape[1]):
                n = c["len"][b, g]
                np.testing.assert_array_equal(f[key][b, g, :n], c[key][b, g, :n], err_msg=f"{what} {key} b{b} g{g}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("with_beta", [True, False])
@pytest.mark.parametrize("S,split_len", [(1, 0), (3, 64)])
def test_paged_decode_stream_matches_flat_oracle(oracle, d, with_beta, S, split_len):
    """Appends across page boundaries up to the budget, then evictions (with the attention's
    candidates), attention after every insertion; three sequences, two kv heads, G = 4."""
    B, Hkv, G, M = 3, 2, 4, 150
    Hq = G * Hkv
    cache = PagedKVCache(B, Hq, Hkv, d, max_pages=3, num_pages=B * Hkv * 3 + 2, M=M, num_splits=S,
                         split_len=split_len, with_beta=with_beta)
    cap = 3 * PAGE
    c = dict(k=np.zeros((B, Hkv, cap, d), np.uint16), v=np.zeros((B, Hkv, cap, d), np.uint16),
             log_beta=np.zeros((B, Hkv, cap), np.float32) if with_beta else None,
             pos=np.zeros((B, Hkv, cap), np.int32), len=np.zeros((B, Hkv), np.int32))
    o = torch.zeros(B, Hq, d, device="cuda")
    lse = torch.zeros(B, Hq, device="cuda")
    g = rng(60, d, S)
    for step in range(230):
        q, kn, vn = normal_bf16(g, (B, Hq, d)), normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d))
        lb = log_beta(g, (B, Hkv))
        t = np.full(B, step, np.int32)
        t[1] = step if step % 7 else -1          # sequence 1 skips some steps (inactive)
        cache.step(dev(q), dev(kn), dev(vn), dev(lb) if with_beta else None, dev(t), o, lse)
        vic = oracle.evict_insert(c, kn, vn, lb if with_beta else None, t, M)
        np.testing.assert_array_equal(host(cache.victim), vic, err_msg=f"step {step}")
        o_ref, l_ref = oracle.decode_attn(q, c["k"], c["v"], c["log_beta"], c["pos"], c["len"], t)
        assert_state_close(host(o), host(lse), o_ref, l_ref, f"step {step}")
        if step % 37 == 0 or step in (63, 64, 65, 149, 150, 229):
            compare(cache, c, f"step {step}")
            check_books(cache.pool)
    assert (host(cache.victim) >= 0).any()
    assert kvb.kvb_get_error() == 0


def test_paged_split_states_match_oracle(oracle):
    B, Hkv, G, d, M, S = 2, 2, 2, 128, 200, 4
    cache = PagedKVCache(B, G * Hkv, Hkv, d, max_pages=4, num_pages=20, M=M, num_splits=S, split_len=64)
    g = rng(61, 0)
    c = dict(k=np.zeros((B, Hkv, 256, d), np.uint16), v=np.zeros((B, Hkv, 256, d), np.uint16),
             log_beta=np.zeros((B, Hkv, 256), np.float32), pos=np.zeros((B, Hkv, 256), np.int32),
             len=np.zeros((B, Hkv), np.int32))
    for step in range(170):
        kn, vn, lb = normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d)), log_beta(g, (B, Hkv))
        t = np.full(B, step, np.int32)
        cache.insert(dev(kn), dev(vn), dev(lb), dev(t))
        oracle.evict_insert(c, kn, vn, lb, t, M)
    q = normal_bf16(g, (B, G * Hkv, d))
    t = np.full(B, 170, np.int32)
    o = torch.zeros(B, G * Hkv, d, device="cuda")
    lse = torch.zeros(B, G * Hkv, device="cuda")
    cache.attend(dev(q), dev(t), o, lse)
    o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(q, c["k"], c["v"], c["log_beta"], c["pos"], c["len"], t,
                                                      num_splits=S, split_len=64, want_parts=True)
    assert_state_close(host(o), host(lse), o_ref, l_ref)
    assert_splits_close(host(cache.o_part), host(cache.lse_part), op_ref, lp_ref)


@pytest.mark.parametrize("d", [64, 128])
def test_paged_compaction_matches_flat_oracle(oracle, d):
    """Removal ranges: inside a page, across pages with a tail longer than the range (overlapping
    move), at the very end, the whole cache, and a no-op; pages past the new length come back."""
    B, Hkv, max_pages = 6, 2, 5
    cap = max_pages * PAGE
    cache = PagedKVCache(B, 2 * Hkv, Hkv, d, max_pages=max_pages, num_pages=B * Hkv * max_pages, M=cap,
                         with_beta=True)
    c = dict(k=np.zeros((B, Hkv, cap, d), np.uint16), v=np.zeros((B, Hkv, cap, d), np.uint16),
             log_beta=np.zeros((B, Hkv, cap), np.float32), pos=np.zeros((B, Hkv, cap), np.int32),
             len=np.zeros((B, Hkv), np.int32))
    g = rng(62, d)
    fill = [300, 300, 257, 64, 190, 10]
    for step in range(max(fill)):
        kn, vn, lb = normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d)), log_beta(g, (B, Hkv))
        t = np.where(step < np.array(fill), step, -1).astype(np.int32)
        cache.insert(dev(kn), dev(vn), dev(lb), dev(t))
        oracle.evict_insert(c, kn, vn, lb, t, cap)
    compare(cache, c, "filled")
    check_books(cache.pool)
    rounds = [(np.array([10, 70, 200, 0, 0, 3]), np.array([20, 100, 57, 64, 0, 7])),
              (np.array([0, 5, 0, 0, 30, 0]), np.array([1, 120, 199, 0, 129, 0]))]
    for rs, rl in rounds:
        rs, rl = rs.astype(np.int32), rl.astype(np.int32)
        cache.compact(dev(rs), dev(rl))
        oracle.compact_blocks(c, rs, rl)
        compare(cache, c, f"after removing {rl.tolist()}")
        check_books(cache.pool)
    assert kvb.kvb_get_error() == 0


def test_paged_pool_exhaustion_flags_error_and_skips_the_insert():
    B, Hkv, d = 2, 1, 64
    cache = PagedKVCache(B, 2, Hkv, d, max_pages=4, num_pages=3, M=256, with_beta=False)
    g = rng(63, 0)
    kvb.kvb_get_error()
    for step in range(129):   # both sequences need a page at 0, 64 and 128: 6 > 3 pages
        kn, vn = normal_bf16(g, (B, Hkv, d)), normal_bf16(g, (B, Hkv, d))
        cache.insert(dev(kn), dev(vn), None, dev(np.full(B, step, np.int32)))
    assert kvb.kvb_get_error() & _lib.DERR_PAGES
    ln = host(cache.len).ravel()
    assert int((-(-ln // PAGE)).sum()) == 3 and ln.max() <= 129
    check_books(cache.pool)


def test_paged_memento_workload_all_sequences(oracle):
    """The memento workload on pages: 64 sequences, every step's append and attention, every
    memento end's removal; the oracle replays the whole batch on the flat layout. Lengths of all
    sequences and the bytes of every compacted sequence are compared at every compaction, the
    whole batch at the end; the page books at every eighth compaction; attention states on a
    sample. The pool holds the schedule's peak page count."""
    w = synth.memento_workload()
    SPLIT_LEN = 512
    S = -(-w.cap // SPLIT_LEN)
    max_pages = -(-w.cap // PAGE)
    cache = PagedKVCache(w.B, w.Hq, w.Hkv, w.d, max_pages=max_pages, num_pages=w.peak_pages(PAGE), M=w.cap,
                         num_splits=S, split_len=SPLIT_LEN, with_beta=False)
    c = dict(k=np.zeros((w.B, w.Hkv, w.cap, w.d), np.uint16), v=np.zeros((w.B, w.Hkv, w.cap, w.d), np.uint16),
             log_beta=None, pos=np.zeros((w.B, w.Hkv, w.cap), np.int32), len=np.zeros((w.B, w.Hkv), np.int32))
    o = torch.zeros(w.B, w.Hq, w.d, device="cuda")
    lse = torch.zeros(w.B, w.Hq, device="cuda")
    watch = [0, 1, 31, 63]
    ends = np.cumsum(w.blk + w.mem, axis=1) - 1
    check_steps = set(np.random.default_rng(7).integers(0, w.steps, 16).tolist())
    for b in watch[:2]:
        for e in ends[b]:
            check_steps.update({int(e), int(e) + 1})
    comp_list = w.compaction_steps().tolist()
    comp_steps = set(comp_list)
    pool = [w.step_inputs(s) for s in range(w.pool)]
    pool_dev = [{key: dev(val) for key, val in inp.items() if key != "t"} for inp in pool]
    peak_used = 0

    def compare_seq(b, what):
        pg = host(cache.pool.table[b])
        ln = c["len"][b]
        kp, vp, pp = cache.pool.k_pages, cache.pool.v_pages, cache.pool.pos_pages
        for g_ in range(w.Hkv):
            n = int(ln[g_])
            ids = torch.from_numpy(pg[g_, : -(-n // PAGE)].astype(np.int64)).cuda()
            for key, t, ref in (("k", kp, c["k"]), ("v", vp, c["v"]), ("pos", pp, c["pos"])):
                got = host(t[ids].reshape(-1, *t.shape[2:])[:n])
                np.testing.assert_array_equal(got, ref[b, g_, :n], err_msg=f"{what} {key} b{b} g{g_}")

    n_compared = 0
    for step in range(w.steps):
        inp = pool[step % w.pool]
        t = np.where(step < w.total, step, -1).astype(np.int32)
        td = dev(t)
        pd = pool_dev[step % w.pool]
        cache.insert(pd["k_new"], pd["v_new"], None, td)
        cache.attend(pd["q"], td, o, lse)
        oracle.evict_insert(c, inp["k_new"], inp["v_new"], None, t, w.cap)
        if step in check_steps:
            o_ref, l_ref = oracle.decode_attn(inp["q"][watch], c["k"][watch], c["v"][watch], None, c["pos"][watch],
                                              c["len"][watch], t[watch])
            assert_state_close(host(o[watch]), host(lse[watch]), o_ref, l_ref, f"step {step}")
        if step in comp_steps:
            peak_used = max(peak_used, cache.pages_in_use())
            rs, rl = w.compaction(step)
            cache.compact(dev(rs), dev(rl))
            oracle.compact_blocks(c, rs, rl)
            np.testing.assert_array_equal(host(cache.len), c["len"], err_msg=f"len after compaction at {step}")
            for b in np.nonzero(rl)[0]:
                compare_seq(int(b), f"compaction at {step}")
                n_compared += 1
            if comp_list.index(step) % 8 == 0:
                check_books(cache.pool)
    assert n_compared == int((w.blk > 0).sum())
    for b in range(w.B):
        compare_seq(b, "end")
    check_books(cache.pool)
    assert peak_used <= w.peak_pages(PAGE)
    assert kvb.kvb_get_error() == 0
