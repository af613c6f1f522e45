"""GPU parity of decode attention over one cache shared by many rows (batch stride 0) with
a fixed split length or one split: kvb_decode_attn then runs its query-batched kernel, which
puts 16 / G rows b of one kv head into the 16 rows of each tensor-core tile and reads every
K/V tile once per block of rows. Each row keeps its own length (a causal prefix) and, with
the retention bias, its own position t. Compared element by element with the oracle, split
states included, on ragged blocks (B not a multiple of 16 / G), empty and inactive rows and
tails that end inside a tile."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200 import _lib
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from gpu_util import dev, host, assert_state_close, assert_splits_close

pytestmark = pytest.mark.gpu


def shared_case(seed, B, G, Hkv, d, cap, bias):
    g = rng(seed, 91)
    Hq = G * Hkv
    q = normal_bf16(g, (B, Hq, d))
    k, v = normal_bf16(g, (1, Hkv, cap, d)), normal_bf16(g, (1, Hkv, cap, d))
    lb = log_beta(g, (1, Hkv, cap)) if bias else None
    pos = np.stack([np.sort(g.permutation(2 * cap)[:cap]) for _ in range(Hkv)])[None].astype(np.int32)
    # consecutive positions over a common prefix: row b sees cap - B + 1 + b slots, plus edge rows
    ln = np.repeat(np.clip(cap - B + 1 + np.arange(B), 0, cap)[:, None], Hkv, axis=1).astype(np.int32)
    ln[0, 0] = 0
    ln[min(1, B - 1), :] = 1
    ln[B // 2, -1] = 63
    t = (2 * cap + np.arange(B)).astype(np.int32)
    t[B - 2] = -1                      # an inactive row
    return q, k, v, lb, pos, ln, t


def run_shared(q, k, v, lb, pos, ln, t, S, split_len):
    B, Hq, d = q.shape
    Hkv, cap = k.shape[1], k.shape[2]
    kd, vd, posd = (dev(x).expand(B, *x.shape[1:]) for x in (k, v, pos))
    lbd = None if lb is None else dev(lb).expand(B, *lb.shape[1:])
    o = torch.full((B, Hq, d), float("nan"), device="cuda")
    lse = torch.full((B, Hq), float("nan"), device="cuda")
    op = lp = None
    if S > 1:
        op, lp = kvb.decode_workspace(B, Hq, d, S)
    kvb.kvb_decode_attn(dev(q), kd, vd, lbd, posd, dev(ln), dev(t), o, lse, num_splits=S, split_len=split_len,
                        o_part=op, lse_part=lp)
    torch.cuda.synchronize()
    return host(o), host(lse), (None if op is None else host(op)), (None if lp is None else host(lp))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bias", [True, False])
@pytest.mark.parametrize("S,split_len", [(1, 0), (3, 96)])
def test_shared_prefix_matches_oracle(oracle, d, G, bias, S, split_len):
    B = 2 * (16 // G) + 3
    q, k, v, lb, pos, ln, t = shared_case(100 + G, B, G, 2, d, 280, bias)
    o, lse, op, lp = run_shared(q, k, v, lb, pos, ln, t, S, split_len)
    o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t, kv_batch_stride=0,
                                                      meta_batch_stride=0, num_splits=S, split_len=split_len,
                                                      want_parts=True)
    assert_state_close(o, lse, o_ref, l_ref, f"d{d} G{G} bias{bias} S{S}")
    assert np.all(lse[B - 2] == -np.inf) and not o[B - 2].any()   # the inactive row
    if S > 1:
        assert_splits_close(op, lp, op_ref, lp_ref, "splits")
    assert kvb.kvb_get_error() == 0


@pytest.mark.parametrize("G", [2, 4, 8])
@pytest.mark.parametrize("bias", [True, False])
@pytest.mark.parametrize("S,split_len", [(1, 0), (3, 96)])
def test_shared_prefix_tensor_core_blocks_match_oracle(oracle, G, bias, S, split_len):
    """At d = 128 with at least 64 query rows the tcgen05 kernel runs (128 rows per unit): two
    full blocks and a ragged third, inactive and empty rows, partial last tiles."""
    BQ = 128 // G
    B = 2 * BQ + 5
    q, k, v, lb, pos, ln, t = shared_case(200 + G, B, G, 2, 128, 280, bias)
    o, lse, op, lp = run_shared(q, k, v, lb, pos, ln, t, S, split_len)
    o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t, kv_batch_stride=0,
                                                      meta_batch_stride=0, num_splits=S, split_len=split_len,
                                                      want_parts=True)
    assert_state_close(o, lse, o_ref, l_ref, f"tcgen05 G{G} bias{bias} S{S}")
    assert np.all(lse[B - 2] == -np.inf) and not o[B - 2].any()
    if S > 1:
        assert_splits_close(op, lp, op_ref, lp_ref, "splits")
    assert kvb.kvb_get_error() == 0


def test_shared_prefix_large_logit_spread(oracle):
    """Keys whose logits grow along the cache (so the running maximum moves by far more than 2^8
    in the exponent, tile after tile): the tcgen05 kernel's lazy rescaling of O must give the
    same softmax."""
    B, G, Hkv, d, cap = 70, 4, 2, 128, 300
    q, k, v, lb, pos, ln, t = shared_case(9, B, G, Hkv, d, cap, True)
    lb[:] = -0.0   # no decay
    from memory_bounded_kv_b200.synth import to_bf16_bits, bf16_bits_to_f32
    kf = bf16_bits_to_f32(k).copy()
    qf = bf16_bits_to_f32(q)
    ramp = np.linspace(0.0, 30.0, cap, dtype=np.float32)   # scale 1/sqrt(d): logit grows ~ 30 * |q0|
    kf[..., 0] = ramp[None, None, :]
    q2 = qf.copy()
    q2[..., 0] = 8.0   # logits span ~21 (30 in log2 units) across the cache
    k, q = to_bf16_bits(kf), to_bf16_bits(q2)
    o, lse, _, _ = run_shared(q, k, v, lb, pos, ln, t, 1, 0)
    o_ref, l_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t, kv_batch_stride=0, meta_batch_stride=0)
    assert_state_close(o, lse, o_ref, l_ref, "large spread")


def test_attention_state_memory_shape(oracle):
    """The self attention of the attention-state-memory workload in the launch configuration the
    bench times: 256 queries at positions 1792..2047 over one 2048-token cache, Hkv 8, G 4, d 128,
    splits of 512 slots."""
    from memory_bounded_kv_b200 import synth
    w = synth.asm_workload()
    o, lse, op, lp = run_shared(w.q, w.k, w.v, None, w.pos, w.len, w.t, 4, 512)
    o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(w.q, w.k, w.v, None, w.pos, w.len, w.t, kv_batch_stride=0,
                                                      meta_batch_stride=0, num_splits=4, split_len=512,
                                                      want_parts=True)
    assert_state_close(o, lse, o_ref, l_ref, "self attention")
    assert_splits_close(op, lp, op_ref, lp_ref, "splits")


def test_shared_prefix_bad_length_flags_error_and_empties_the_row():
    q, k, v, lb, pos, ln, t = shared_case(7, 9, 4, 2, 128, 200, True)
    ln[3, 1] = 201                     # above the capacity
    kvb.kvb_get_error()
    o, lse, _, _ = run_shared(q, k, v, lb, pos, ln, t, 1, 0)
    assert kvb.kvb_get_error() & _lib.DERR_LEN
    assert np.all(lse[3, 4:] == -np.inf) and not o[3, 4:].any()
    assert np.all(np.isfinite(lse[3, :4]))


@pytest.mark.parametrize("B", [11, 40])   # the mma.sync kernel (44 rows) and the tcgen05 kernel (160 rows)
def test_shared_prefix_bounded_wait_runs_out(oracle, B):
    q, k, v, lb, pos, ln, t = shared_case(8, B, 4, 2, 128, 200, False)
    kvb.kvb_get_error()
    kvb.kvb_test_withhold_next_decode(20_000)
    o, lse, _, lp = run_shared(q, k, v, lb, pos, ln, t, 2, 128)
    assert kvb.kvb_get_error() & _lib.DERR_TIMEOUT
    assert np.all(lse == -np.inf) and not o.any() and np.all(lp == -np.inf)
    # one launch only: the same call now matches the oracle
    o, lse, _, _ = run_shared(q, k, v, lb, pos, ln, t, 2, 128)
    assert kvb.kvb_get_error() == 0
    o_ref, l_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t, kv_batch_stride=0, meta_batch_stride=0)
    assert_state_close(o, lse, o_ref, l_ref, "after the timeout")
