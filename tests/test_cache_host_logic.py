"""Host logic of BoundedKVCache.step (no GPU): which launches a decode step makes. One launch
(kvb_decode_step) when the cache is known to be full and the last operation was an attention
that left eviction records; else budget enforcement + insertion, then attention. The fused step
reads the record buffer the previous attention wrote and writes the other one, and the roles swap
every step. The library calls are replaced by recorders; the tensors stay on the CPU."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200.cache as cm

B, Hq, Hkv, d, cap, M = 2, 8, 2, 64, 16, 16


@pytest.fixture
def calls(monkeypatch):
    log = []
    monkeypatch.setattr(cm, "kvb_evict_insert",
                        lambda *a, **k: log.append(("insert", k.get("cand"))))
    monkeypatch.setattr(cm, "kvb_decode_attn",
                        lambda *a, **k: log.append(("attend", k.get("evict_cand"))))
    monkeypatch.setattr(cm, "kvb_decode_step",
                        lambda *a, **k: log.append(("step", a[13], a[14])))   # cand_in, cand_out
    monkeypatch.setattr(cm, "kvb_compact_blocks", lambda *a, **k: log.append(("compact",)))
    return log


def make_cache(lens, with_beta=True):
    k = np.zeros((B, Hkv, cap, d), np.uint16)
    lb = np.zeros((B, Hkv, cap), np.float32) if with_beta else None
    pos = np.zeros((B, Hkv, cap), np.int32)
    return cm.BoundedKVCache.from_host(k, k, lb, pos, np.asarray(lens, np.int32), Hq, M, num_splits=2,
                                       device="cpu")


def step_inputs():
    bf = torch.bfloat16
    return (torch.zeros(B, Hq, d, dtype=bf), torch.zeros(B, Hkv, d, dtype=bf), torch.zeros(B, Hkv, d, dtype=bf),
            torch.zeros(B, Hkv), torch.zeros(B, dtype=torch.int32), torch.zeros(B, Hq, d), torch.zeros(B, Hq))


def do_step(c):
    q, kn, vn, lbn, t, o, lse = step_inputs()
    c.step(q, kn, vn, lbn, t, o, lse)


def test_a_full_cache_fuses_every_step_after_the_first(calls):
    c = make_cache(np.full((B, Hkv), M))
    assert c.full
    do_step(c)   # no records yet: the scan, then the attention that leaves them
    assert [x[0] for x in calls] == ["insert", "attend"]
    assert calls[0][1] is None and calls[1][1] is not None
    written = calls[1][1]
    do_step(c)
    do_step(c)
    kinds = [x[0] for x in calls]
    assert kinds == ["insert", "attend", "step", "step"]
    # each fused step reads what the step before it wrote and writes the other buffer
    assert calls[2][1] is written and calls[2][2] is not written
    assert calls[3][1] is calls[2][2] and calls[3][2] is written
    assert c.cand_valid


def test_a_cache_below_its_budget_never_fuses(calls):
    lens = np.full((B, Hkv), M)
    lens[1, 0] = M - 3
    c = make_cache(lens)
    assert not c.full
    for _ in range(3):
        do_step(c)
    assert [x[0] for x in calls] == ["insert", "attend"] * 3
    # the insertion uses the records of the attention just before it
    assert calls[2][1] is calls[1][1] and calls[4][1] is calls[3][1]


def test_compaction_and_attention_without_records_end_the_fused_steps(calls):
    c = make_cache(np.full((B, Hkv), M))
    do_step(c)
    do_step(c)
    c.compact(torch.zeros(B, dtype=torch.int32), torch.zeros(B, dtype=torch.int32))
    assert not c.full and not c.cand_valid
    do_step(c)
    assert [x[0] for x in calls] == ["insert", "attend", "step", "compact", "insert", "attend"]
    # an attention that leaves no records (plain scoring on a retention cache) makes the
    # records stale for the next insertion
    c2 = make_cache(np.full((B, Hkv), M))
    calls.clear()
    q, kn, vn, lbn, t, o, lse = step_inputs()
    c2.attend(q, t, o, lse, use_beta=False)
    assert calls == [("attend", None)] and not c2.cand_valid
    do_step(c2)
    assert [x[0] for x in calls] == ["attend", "insert", "attend"] and calls[1][1] is None
