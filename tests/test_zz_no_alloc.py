"""kvb_decode_attn_noalloc: the decode-attention entry point for callers that cannot
hand the library scratch device memory (for instance a plugin running inside a serving
process that owns every device allocation, or a decode path that must never call
cudaMalloc because it would synchronize the device or fail when memory is reserved).

It keeps the split states in a fixed array inside the library. These tests call it
through the C ABI and compare it with kvb_decode_attn (which takes caller scratch) and
with the CPU oracle on two calls in a row, with different shapes so the second call reuses
an array that the first one left dirty. This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200 import _lib
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from gpu_util import dev, host, assert_state_close

pytestmark = pytest.mark.gpu


def _host_case(seed, B, Hq, Hkv, d, cap, fill):
    g = rng(seed, 77)
    q, k, v = normal_bf16(g, (B, Hq, d)), normal_bf16(g, (B, Hkv, cap, d)), normal_bf16(g, (B, Hkv, cap, d))
    lb = log_beta(g, (B, Hkv, cap))
    pos = np.tile(np.arange(cap, dtype=np.int32), (B, Hkv, 1))
    ln = np.minimum(cap, (fill * cap + g.integers(0, cap, (B, Hkv)) // 4)).astype(np.int32)
    t = np.full(B, cap + 3, np.int32)
    return q, k, v, lb, pos, ln, t


def _case(seed, B, Hq, Hkv, d, cap, fill):
    return [dev(x) for x in _host_case(seed, B, Hq, Hkv, d, cap, fill)]


def _both(args, S):
    q, k, v, lb, pos, ln, t = args
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    o_ref = torch.zeros(B, Hq, d, device="cuda")
    l_ref = torch.zeros(B, Hq, device="cuda")
    op, lp = kvb.decode_workspace(B, Hq, d, S)
    kvb.kvb_decode_attn(q, k, v, lb, pos, ln, t, o_ref, l_ref, num_splits=S, o_part=op, lse_part=lp)
    o = torch.full((B, Hq, d), float("nan"), device="cuda")
    lse = torch.full((B, Hq), float("nan"), device="cuda")
    kvb.kvb_decode_attn_noalloc(q, k, v, lb, pos, ln, t, o, lse, num_splits=S)
    torch.cuda.synchronize()
    return host(o), host(lse), host(o_ref), host(l_ref)


def test_noalloc_matches_scratch_entry_point_on_two_calls_in_a_row(oracle):
    # call 1: Qwen3-8B-shaped heads, 16 splits (8.4 MB of split states at B=32 fits the 16 MiB array)
    h1 = _host_case(1, 32, 32, 8, 128, 4096, 0.75)
    o, lse, o_ref, l_ref = _both([dev(x) for x in h1], 16)
    assert_state_close(o, lse, o_ref, l_ref, "call 1")
    assert_state_close(o, lse, *oracle.decode_attn(*h1), "call 1 against the oracle")
    # call 2: a different shape, so its lse_part and o_part rows overlay different offsets of the
    # array that call 1 left dirty
    h2 = _host_case(2, 5, 16, 2, 64, 700, 0.5)
    o, lse, o_ref, l_ref = _both([dev(x) for x in h2], 7)
    assert_state_close(o, lse, o_ref, l_ref, "call 2")
    assert_state_close(o, lse, *oracle.decode_attn(*h2), "call 2 against the oracle")
    assert kvb.kvb_get_error() == 0


def test_noalloc_single_split_and_repeat():
    args = _case(3, 3, 8, 2, 128, 300, 0.9)
    for _ in range(2):
        o, lse, o_ref, l_ref = _both(args, 1)
        assert_state_close(o, lse, o_ref, l_ref, "S=1")


def test_noalloc_rejects_problems_larger_than_its_array():
    q, k, v, lb, pos, ln, t = _case(4, 8, 32, 8, 128, 256, 1.0)
    o = torch.zeros(8, 32, 128, device="cuda")
    S = 1024   # 8*32*1024*129*4 bytes of split states > 16 MiB
    assert 8 * 32 * S * 128 * 4 > _lib.NOALLOC_SCRATCH_BYTES
    with pytest.raises(kvb.KvbError) as e:
        kvb.kvb_decode_attn_noalloc(q, k, v, lb, pos, ln, t, o, num_splits=S)
    assert e.value.status == _lib.KVB_EINVAL
    # caller scratch is refused: the array is the only scratch this entry point uses
    a = _lib.AttnArgs(q=q.data_ptr(), q_stride_b=32 * 128, q_stride_h=128, k=k.data_ptr(), v=v.data_ptr(),
                      kv_stride_b=8 * 256 * 128, kv_stride_h=256 * 128, len=ln.data_ptr(), B=8, Hq=32, Hkv=8,
                      d=128, cap=256, num_splits=2, o_part=o.data_ptr(), lse_part=o.data_ptr(),
                      counters=ln.data_ptr(), o=o.data_ptr())
    import ctypes
    assert _lib.lib().kvb_decode_attn_noalloc(ctypes.byref(a), None) == _lib.KVB_EINVAL
