"""Raw dump and reload of a decode step (memory_bounded_kv_b200.state), on the CPU: every tensor
comes back bit for bit with its dtype and shape, the cache is rebuilt with the dumped sizes, and
damaged dumps are refused instead of being read short."""
import json
import os

import numpy as np
import pytest
import torch

from memory_bounded_kv_b200 import state
from memory_bounded_kv_b200.cache import BoundedKVCache
from memory_bounded_kv_b200.synth import normal_bf16, log_beta, rng


def _filled_cache(with_beta):
    B, Hq, Hkv, d, cap, M = 2, 8, 2, 64, 96, 80
    c = BoundedKVCache(B, Hq, Hkv, d, cap, M, num_splits=3, split_len=32, with_beta=with_beta, device="cpu")
    g = rng(5, int(with_beta))
    c.k.copy_(torch.from_numpy(normal_bf16(g, (B, Hkv, cap, d)).view(np.int16)).view(torch.bfloat16))
    c.v.copy_(torch.from_numpy(normal_bf16(g, (B, Hkv, cap, d)).view(np.int16)).view(torch.bfloat16))
    if with_beta:
        c.log_beta.copy_(torch.from_numpy(log_beta(g, (B, Hkv, cap))))
    c.pos.copy_(torch.from_numpy(g.permutation(cap * B * Hkv).reshape(B, Hkv, cap).astype(np.int32)))
    c.len.copy_(torch.tensor([[80, 17], [0, 80]], dtype=torch.int32))
    return c


def _bits(x):
    x = x.detach().cpu().contiguous()
    return x.view(torch.int16).numpy() if x.dtype == torch.bfloat16 else x.numpy()


@pytest.mark.parametrize("with_beta", [True, False])
def test_flat_step_round_trips_bit_for_bit(tmp_path, with_beta):
    c = _filled_cache(with_beta)
    g = rng(6)
    inputs = dict(q=normal_bf16(g, (c.B, c.Hq, c.d)),                       # numpy bf16 patterns
                  k_new=torch.from_numpy(normal_bf16(g, (c.B, c.Hkv, c.d)).view(np.int16)).view(torch.bfloat16),
                  v_new=normal_bf16(g, (c.B, c.Hkv, c.d)),
                  log_beta_new=log_beta(g, (c.B, c.Hkv)) if with_beta else None,
                  t=np.array([1000, 1001], np.int32))
    path = str(tmp_path / "step")
    state.dump_step(path, c, inputs, extra_meta={"workload": "unit test", "step": 7})
    doc = json.load(open(os.path.join(path, "state.json")))
    assert doc["meta"]["kind"] == "flat" and doc["meta"]["extra"]["step"] == 7
    assert ("log_beta" in doc["tensors"]) == with_beta
    assert ("in_log_beta_new" in doc["tensors"]) == with_beta

    c2, inp2, meta = state.load_step(path, device="cpu")
    for name in ("k", "v", "pos", "len") + (("log_beta",) if with_beta else ()):
        a, b = getattr(c, name), getattr(c2, name)
        assert a.dtype == b.dtype and a.shape == b.shape, name
        np.testing.assert_array_equal(_bits(a), _bits(b), err_msg=name)
    assert (c2.log_beta is None) == (not with_beta)
    assert (c2.M, c2.cap, c2.num_splits, c2.split_len) == (c.M, c.cap, c.num_splits, c.split_len)
    np.testing.assert_array_equal(_bits(inp2["q"]).view(np.uint16), inputs["q"])
    np.testing.assert_array_equal(_bits(inp2["k_new"]), _bits(inputs["k_new"]))
    np.testing.assert_array_equal(_bits(inp2["v_new"]).view(np.uint16), inputs["v_new"])
    np.testing.assert_array_equal(inp2["t"].numpy(), inputs["t"])
    assert inp2["q"].dtype == torch.bfloat16 and inp2["t"].dtype == torch.int32
    if with_beta:
        np.testing.assert_array_equal(inp2["log_beta_new"].numpy(), inputs["log_beta_new"])
    else:
        assert "log_beta_new" not in inp2


def test_damaged_dumps_are_refused(tmp_path):
    c = _filled_cache(True)
    path = str(tmp_path / "s")
    state.dump_step(path, c, dict(t=np.zeros(2, np.int32)))
    with open(os.path.join(path, "k.bin"), "r+b") as f:      # one element short
        f.truncate(os.path.getsize(os.path.join(path, "k.bin")) - 2)
    with pytest.raises(ValueError, match="k.bin"):
        state.load_step(path, device="cpu")

    path2 = str(tmp_path / "s2")
    state.dump_step(path2, c, {})
    doc = json.load(open(os.path.join(path2, "state.json")))
    doc["format"] = 99
    json.dump(doc, open(os.path.join(path2, "state.json"), "w"))
    with pytest.raises(ValueError, match="format"):
        state.load(path2, device="cpu")

    path3 = str(tmp_path / "s3")
    state.dump_step(path3, c, {})
    doc = json.load(open(os.path.join(path3, "state.json")))
    doc["meta"]["cap"] = 128                                  # sizes that do not match the files
    json.dump(doc, open(os.path.join(path3, "state.json"), "w"))
    with pytest.raises(ValueError, match="k: dumped"):
        state.load_step(path3, device="cpu")


def test_unknown_inputs_and_dtypes_are_refused(tmp_path):
    c = _filled_cache(False)
    with pytest.raises(ValueError, match="unknown step inputs"):
        state.dump_step(str(tmp_path / "a"), c, dict(qq=np.zeros(3, np.int32)))
    with pytest.raises(TypeError):
        state.save(str(tmp_path / "b"), dict(x=np.zeros(3, np.float16)), {})
