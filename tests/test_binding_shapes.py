"""The Python binding checks every tensor's shape before anything reaches the library: the
C ABI takes plain pointers and cannot see buffer sizes, so an undersized output or workspace
would otherwise be written past its end. These tests use CPU tensors (no GPU): the shape
checks run before the device checks, so a wrong shape raises ValueError first."""
import pytest
import torch

import memory_bounded_kv_b200 as kvb

B, Hq, Hkv, d, cap, S = 2, 8, 2, 64, 32, 4


def decode_args():
    bf = torch.bfloat16
    return dict(q=torch.zeros(B, Hq, d, dtype=bf), k=torch.zeros(B, Hkv, cap, d, dtype=bf),
                v=torch.zeros(B, Hkv, cap, d, dtype=bf), log_beta=torch.zeros(B, Hkv, cap),
                pos=torch.zeros(B, Hkv, cap, dtype=torch.int32), len=torch.zeros(B, Hkv, dtype=torch.int32),
                t=torch.zeros(B, dtype=torch.int32), o=torch.zeros(B, Hq, d), lse=torch.zeros(B, Hq))


def call_decode(entry=kvb.kvb_decode_attn, num_splits=1, **over):
    a = decode_args()
    extra = {k: over.pop(k) for k in ("o_part", "lse_part") if k in over}
    a.update(over)
    entry(a["q"], a["k"], a["v"], a["log_beta"], a["pos"], a["len"], a["t"], a["o"], a["lse"],
          num_splits=num_splits, **extra)


def test_well_shaped_cpu_tensors_pass_the_shape_checks():
    # shapes are fine, so the next check (CUDA tensors) is the one that refuses
    with pytest.raises(TypeError, match="CUDA"):
        call_decode()


@pytest.mark.parametrize("entry", [kvb.kvb_decode_attn, kvb.kvb_decode_attn_noalloc])
@pytest.mark.parametrize("name,shape", [
    ("o", (B, Hq - 1, d)), ("o", (B - 1, Hq, d)), ("lse", (B, Hq - 1)), ("len", (B - 1, Hkv)), ("t", (B + 1,)),
    ("log_beta", (B, Hkv, cap - 1)), ("pos", (B, 1, cap)), ("v", (B, Hkv, cap - 8, d)),
])
def test_decode_rejects_a_wrong_shape_before_any_launch(entry, name, shape):
    bad = torch.zeros(shape, dtype=decode_args()[name].dtype)
    with pytest.raises(ValueError, match=name):
        call_decode(entry, **{name: bad})


def test_decode_split_workspace_must_match_num_splits():
    op, lp = torch.zeros(B, Hq, S, d), torch.zeros(B, Hq, S)
    with pytest.raises(ValueError, match="o_part"):   # a workspace for S splits used with 2S
        call_decode(num_splits=2 * S, o_part=op, lse_part=torch.zeros(B, Hq, 2 * S))
    with pytest.raises(ValueError, match="lse_part"):
        call_decode(num_splits=S, o_part=op, lse_part=torch.zeros(B, Hq, S - 1))
    with pytest.raises(ValueError, match="o_part"):   # several splits need the split-state buffers
        call_decode(num_splits=S)


def test_evict_insert_and_compaction_check_shapes():
    a = decode_args()
    kn, vn = torch.zeros(B, Hkv, d, dtype=torch.bfloat16), torch.zeros(B, Hkv, d, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="k_new"):
        kvb.kvb_evict_insert(a["k"], a["v"], a["log_beta"], a["pos"], a["len"], kn[:1], vn, torch.zeros(B, Hkv),
                             a["t"], cap)
    with pytest.raises(ValueError, match="victim"):
        kvb.kvb_evict_insert(a["k"], a["v"], a["log_beta"], a["pos"], a["len"], kn, vn, torch.zeros(B, Hkv),
                             a["t"], cap, torch.zeros(B, dtype=torch.int32))
    with pytest.raises(ValueError, match="rm_len"):
        kvb.kvb_compact_blocks(a["k"], a["v"], a["pos"], None, a["len"], torch.zeros(B, dtype=torch.int32),
                               torch.zeros(B - 1, dtype=torch.int32))


def test_decode_step_checks_the_new_rows_before_any_launch():
    a = decode_args()
    bf = torch.bfloat16
    kn, vn = torch.zeros(B, Hkv, d, dtype=bf), torch.zeros(B, Hkv, d, dtype=bf)
    lbn = torch.zeros(B, Hkv)
    cand = torch.zeros(B * Hkv * 2, dtype=torch.int64)

    def step(**over):
        x = dict(k_new=kn, v_new=vn, log_beta_new=lbn, cand_in=cand, cand_out=cand, victim=None)
        x.update(over)
        kvb.kvb_decode_step(a["q"], a["k"], a["v"], a["log_beta"], a["pos"], a["len"], a["t"], a["o"], a["lse"],
                            x["k_new"], x["v_new"], x["log_beta_new"], cap, x["cand_in"], x["cand_out"],
                            victim=x["victim"])

    with pytest.raises(TypeError, match="CUDA"):   # well shaped: the device check refuses
        step()
    with pytest.raises(ValueError, match="k_new"):
        step(k_new=kn[:1])
    with pytest.raises(ValueError, match="v_new"):
        step(v_new=torch.zeros(B, Hkv, d - 8, dtype=bf))
    with pytest.raises(ValueError, match="log_beta_new"):
        step(log_beta_new=torch.zeros(B, Hkv + 1))
    with pytest.raises(ValueError, match="log_beta_new"):   # a retention cache needs the new log beta
        step(log_beta_new=None)
    with pytest.raises(ValueError, match="victim"):
        step(victim=torch.zeros(B * Hkv - 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="cand"):
        step(cand_in=None)
