"""The oracle's parallel driver (oracle_decode_steps_threads) spreads independent
(sequence, kv head) units over threads, each running the serial oracle functions on
one unit's slice. Pinned here against those serial functions called step by step over
the whole batch: victims, every cache byte, and the attention state must be identical
bit for bit (same arithmetic, same order within a unit)."""
import numpy as np
import pytest

from memory_bounded_kv_b200 import synth


def serial(w, c, steps, with_q=True, with_kv=True):
    vic, o, lse = [], None, None
    for s in range(steps):
        x = w.step_inputs(s)
        vic.append(oracle_mod.evict_insert(c, x["k_new"] if with_kv else None, x["v_new"] if with_kv else None,
                                           x["log_beta_new"], x["t"], w.M))
        if with_q:
            o, lse = oracle_mod.decode_attn(x["q"], c["k"], c["v"], c["log_beta"], c["pos"], c["len"], x["t"])
    return np.stack(vic), o, lse


def stacked(w, steps):
    xs = [w.step_inputs(s) for s in range(steps)]
    return {key: np.stack([x[key] for x in xs]) for key in xs[0]}


def cache_of(w):
    return dict(k=w.k.copy(), v=w.v.copy(), log_beta=w.log_beta.copy(), pos=w.pos.copy(), len=w.len.copy())


oracle_mod = None


@pytest.fixture(autouse=True)
def _oracle(oracle):
    global oracle_mod
    oracle_mod = oracle


@pytest.mark.parametrize("nthreads", [1, 3, 0])
def test_threaded_decode_steps_equal_the_serial_oracle(nthreads):
    w = synth.decode_workload(1, prefill=200)   # B=1, 8/2 heads, d 64: appends, then evictions
    w.B = 1
    steps = 90
    c1, c2 = cache_of(w), cache_of(w)
    v1, o1, l1 = serial(w, c1, steps)
    x = stacked(w, steps)
    v2, o2, l2 = oracle_mod.decode_steps_threads(c2, x["q"], x["k_new"], x["v_new"], x["log_beta_new"], x["t"], w.M,
                                                 nthreads)
    np.testing.assert_array_equal(v1, v2)
    assert (v1 >= 0).any() and (v1 < 0).any()
    for key in ("k", "v", "log_beta", "pos", "len"):
        np.testing.assert_array_equal(c1[key], c2[key], err_msg=key)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_threaded_stream_without_attention_or_kv():
    """The long-context build's mode: only log beta and pos stream through eviction."""
    w = synth.decode_workload(2, B=3, prefill=64)
    w.M = 64
    steps = 50
    c1, c2 = cache_of(w), cache_of(w)
    v1, _, _ = serial(w, c1, steps, with_q=False, with_kv=False)
    x = stacked(w, steps)
    v2, o2, l2 = oracle_mod.decode_steps_threads(c2, None, None, None, x["log_beta_new"], x["t"], w.M, 4)
    assert o2 is None and l2 is None
    np.testing.assert_array_equal(v1, v2)
    for key in ("k", "v", "log_beta", "pos", "len"):
        np.testing.assert_array_equal(c1[key], c2[key], err_msg=key)
