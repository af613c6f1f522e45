"""GPU parity of kvb_decode_attn against the oracle on small seeded inputs that
span several tiles and ragged tails: every (d, G), with and without the
retention bias, one and many splits, fixed split lengths, bf16 output, a
shared cache (batch stride 0), inactive rows, empty caches and bad lengths."""
import numpy as np
import pytest
import torch

import memory_bounded_kv_b200 as kvb
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng
from gpu_util import dev, host, assert_state_close, assert_splits_close, bf16_round

pytestmark = pytest.mark.gpu


def make_case(seed, B, Hq, Hkv, d, cap, lens, bias=True):
    g = rng(seed, 42)
    q = normal_bf16(g, (B, Hq, d))
    k = normal_bf16(g, (B, Hkv, cap, d))
    v = normal_bf16(g, (B, Hkv, cap, d))
    lb = log_beta(g, (B, Hkv, cap)) if bias else None
    t = np.full(B, 2 * cap + 5, np.int32)
    pos = np.stack([np.stack([np.sort(g.permutation(2 * cap)[:cap]) for _ in range(Hkv)]) for _ in range(B)])
    pos = pos.astype(np.int32)
    ln = np.asarray(lens, np.int32).reshape(B, Hkv)
    return q, k, v, lb, pos, ln, t


def run_gpu(q, k, v, lb, pos, ln, t, S=1, split_len=0, out_bf16=False, kv_shared=False):
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    qd, kd, vd = dev(q), dev(k), dev(v)
    lbd = None if lb is None else dev(lb)
    posd = dev(pos)
    if kv_shared:
        kd = kd.expand(B, *kd.shape[1:])
        vd = vd.expand(B, *vd.shape[1:])
        posd = posd.expand(B, *posd.shape[1:])
        if lbd is not None:
            lbd = lbd.expand(B, *lbd.shape[1:])
    o = torch.zeros(B, Hq, d, dtype=torch.bfloat16 if out_bf16 else torch.float32, device="cuda")
    lse = torch.zeros(B, Hq, dtype=torch.float32, device="cuda")
    op = lp = None
    if S > 1:
        op, lp = kvb.decode_workspace(B, Hq, d, S)
    kvb.kvb_decode_attn(qd, kd, vd, lbd, posd, dev(ln), None if t is None else dev(t), o, lse, num_splits=S,
                        split_len=split_len, o_part=op, lse_part=lp)
    torch.cuda.synchronize()
    res = dict(o=host(o.float()) if out_bf16 else host(o), lse=host(lse))
    if op is not None:
        res["o_part"], res["lse_part"] = host(op), host(lp)
    return res


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bias", [True, False])
@pytest.mark.parametrize("S", [1, 3, 16])
def test_decode_matches_oracle(oracle, d, G, bias, S):
    Hkv = 2
    B, Hq, cap = 3, Hkv * G, 300
    lens = [[300, 1], [0, 257], [64, 129]]   # full, single, empty, ragged tails
    q, k, v, lb, pos, ln, t = make_case(d * 10 + G + 3 * bias + S, B, Hq, Hkv, d, cap, lens, bias)
    res = run_gpu(q, k, v, lb, pos, ln, t if bias else None, S=S)
    o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t if bias else None, num_splits=S,
                                                      want_parts=True)
    assert_state_close(res["o"], res["lse"], o_ref, l_ref, "final")
    if S > 1:
        assert_splits_close(res["o_part"], res["lse_part"], op_ref, lp_ref, "splits")


@pytest.mark.parametrize("S,split_len", [(4, 128), (8, 40), (40, 8), (1024, 1)])
def test_fixed_split_length(oracle, S, split_len):
    q, k, v, lb, pos, ln, t = make_case(7, 2, 8, 2, 128, 320, [[320, 100], [7, 0]])
    ln = np.minimum(ln, S * split_len).astype(np.int32)
    res = run_gpu(q, k, v, lb, pos, ln, t, S=S, split_len=split_len)
    o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t, num_splits=S, split_len=split_len,
                                                      want_parts=True)
    assert_state_close(res["o"], res["lse"], o_ref, l_ref, "final")
    assert_splits_close(res["o_part"], res["lse_part"], op_ref, lp_ref, "splits")


def test_bf16_output_against_rounded_oracle(oracle):
    q, k, v, lb, pos, ln, t = make_case(8, 2, 16, 4, 128, 200, [[200, 3, 150, 77], [1, 2, 200, 199]])
    res = run_gpu(q, k, v, lb, pos, ln, t, S=4, out_bf16=True)
    o_ref, l_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    assert_state_close(res["o"], res["lse"], bf16_round(o_ref), l_ref, "bf16 out")


def test_shared_cache_batch_stride_zero(oracle):
    B, Hq, Hkv, d, cap = 6, 8, 2, 128, 500
    q, k, v, lb, pos, _, t = make_case(9, B, Hq, Hkv, d, cap, [[cap, cap]] * B)
    ln = np.array([[1, 2], [100, 499], [500, 500], [0, 250], [64, 65], [63, 7]], np.int32)
    res = run_gpu(q, k[:1], v[:1], lb[:1], pos[:1], ln, t, S=5, kv_shared=True)
    o_ref, l_ref = oracle.decode_attn(q, k[:1], v[:1], lb[:1], pos[:1], ln, t, kv_batch_stride=0,
                                      meta_batch_stride=0)
    assert_state_close(res["o"], res["lse"], o_ref, l_ref, "shared cache")


def test_inactive_rows_are_empty(oracle):
    q, k, v, lb, pos, ln, t = make_case(10, 3, 8, 2, 64, 100, [[100, 100]] * 3)
    t[1] = -1
    res = run_gpu(q, k, v, lb, pos, ln, t, S=2)
    assert np.all(res["lse"][1] == -np.inf) and not res["o"][1].any()
    o_ref, l_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    assert_state_close(res["o"], res["lse"], o_ref, l_ref, "inactive")


def test_bad_length_sets_device_error_and_empty_state():
    q, k, v, lb, pos, ln, t = make_case(11, 2, 8, 2, 128, 64, [[64, 65], [10, 10]])
    kvb.kvb_get_error()  # clear
    res = run_gpu(q, k, v, lb, pos, ln, t, S=2)
    bits = kvb.kvb_get_error()
    assert bits & 1, bits
    assert np.all(res["lse"][0, 4:] == -np.inf) and np.all(np.isfinite(res["lse"][0, :4]))
    assert kvb.kvb_get_error() == 0  # cleared


def test_split_len_overflow_sets_device_error():
    q, k, v, lb, pos, ln, t = make_case(12, 1, 4, 1, 128, 64, [[64]])
    kvb.kvb_get_error()
    res = run_gpu(q, k, v, lb, pos, ln, t, S=2, split_len=16)
    assert kvb.kvb_get_error() & 2
    assert np.all(res["lse"] == -np.inf)


def test_repeated_calls_reuse_workspace(oracle):
    q, k, v, lb, pos, ln, t = make_case(13, 2, 32, 8, 128, 256, [[256] * 8, [100] * 8])
    B, Hq, d = q.shape
    qd, kd, vd, lbd, posd, lnd, td = map(dev, (q, k, v, lb, pos, ln, t))
    op, lp = kvb.decode_workspace(B, Hq, d, 7)
    outs = []
    for _ in range(5):
        o = torch.empty(B, Hq, d, device="cuda")
        lse = torch.empty(B, Hq, device="cuda")
        kvb.kvb_decode_attn(qd, kd, vd, lbd, posd, lnd, td, o, lse, num_splits=7, o_part=op, lse_part=lp)
        outs.append((host(o), host(lse)))
    for o, lse in outs[1:]:
        np.testing.assert_array_equal(o, outs[0][0])
        np.testing.assert_array_equal(lse, outs[0][1])
    o_ref, l_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t)
    assert_state_close(outs[0][0], outs[0][1], o_ref, l_ref)


def test_explicit_scale(oracle):
    q, k, v, lb, pos, ln, t = make_case(14, 1, 4, 1, 64, 90, [[90]])
    B, Hq, d = q.shape
    o = torch.zeros(B, Hq, d, device="cuda")
    lse = torch.zeros(B, Hq, device="cuda")
    kvb.kvb_decode_attn(dev(q), dev(k), dev(v), dev(lb), dev(pos), dev(ln), dev(t), o, lse, scale=0.3)
    o_ref, l_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t, scale=0.3)
    assert_state_close(host(o), host(lse), o_ref, l_ref)


def test_host_rejects_bad_layout():
    q, k, v, lb, pos, ln, t = make_case(15, 1, 4, 1, 64, 16, [[16]])
    o = torch.zeros(1, 4, 64, device="cuda")
    with pytest.raises(ValueError):   # num_splits > 1 without split-state buffers
        kvb.kvb_decode_attn(dev(q), dev(k), dev(v), dev(lb), dev(pos), dev(ln), dev(t), o, num_splits=2)
    with pytest.raises(kvb.KvbError):   # q not 16-byte aligned: refused by the library
        qd = torch.empty(q.size + 8, dtype=torch.bfloat16, device="cuda")[1:1 + q.size].view(q.shape)
        kvb.kvb_decode_attn(qd, dev(k), dev(v), dev(lb), dev(pos), dev(ln), dev(t), o)


@pytest.mark.parametrize("d,G,S", [(128, 4, 8), (128, 4, 5), (64, 8, 2), (128, 8, 16), (64, 1, 3)])
def test_equal_splits_many_rows(oracle, d, G, S):
    """Equal splits (split_len 0) over many (b, g) rows (up to 4096 units: the persistent CTAs
    take several in turn); lengths below S leave empty splits, length 0 empty rows. Final states
    and every split's state against the oracle."""
    Hkv = 2 if G == 8 else 8
    B, Hq, cap = 64, Hkv * G, 130
    g = rng(77, d + G + S)
    lens = g.integers(0, cap + 1, (B, Hkv))
    lens[0, :] = [0, 1] + [2] * (Hkv - 2)
    lens[1, 0], lens[2, 0] = S - 1, cap
    q, k, v, lb, pos, ln, t = make_case(d + 3 * G + 7 * S, B, Hq, Hkv, d, cap, lens)
    kvb.kvb_get_error()   # clear
    res = run_gpu(q, k, v, lb, pos, ln, t, S=S)
    o_ref, l_ref, op_ref, lp_ref = oracle.decode_attn(q, k, v, lb, pos, ln, t, num_splits=S, want_parts=True)
    assert_state_close(res["o"], res["lse"], o_ref, l_ref, "final")
    assert_splits_close(res["o_part"], res["lse_part"], op_ref, lp_ref, "splits")
    assert kvb.kvb_get_error() == 0
