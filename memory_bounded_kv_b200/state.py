"""Raw dump and reload of a decode step: the cache state before it and the step's inputs.

A directory holds one `<name>.bin` per tensor (its bytes, little-endian, C order; bf16 as its
16-bit patterns) and `state.json`, which gives each tensor's dtype and shape and the cache's
sizes. `replay_step` runs the dumped step once through the library on a cache rebuilt from the
files, so a step that went wrong in a long stream can be re-run alone, compared with any other
implementation of the same step, or bisected without the stream that led to it.

Flat caches (BoundedKVCache) and paged caches (PagedKVCache) are both covered; the tensors are
the ones the kernels read: K, V, log beta (absent for beta = 1), pos, len, plus the block table
and the free-page stack for pages. The step's inputs are q, k_new, v_new, log_beta_new (absent
for beta = 1), t, and optionally a compaction (rm_start, rm_len) applied after the attention.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

_FORMAT = 1
_DTYPES = {torch.bfloat16: "bf16", torch.float32: "f32", torch.int32: "i32", torch.int64: "i64"}
_NP = {"bf16": np.uint16, "f32": np.float32, "i32": np.int32, "i64": np.int64}
_TORCH = {v: k for k, v in _DTYPES.items()}


def _host_bytes(x) -> tuple[str, tuple, bytes]:
    if isinstance(x, np.ndarray):
        a = np.ascontiguousarray(x)
        kind = {np.dtype(np.uint16): "bf16", np.dtype(np.float32): "f32", np.dtype(np.int32): "i32",
                np.dtype(np.int64): "i64"}.get(a.dtype)
        if kind is None:
            raise TypeError(f"cannot dump an array of dtype {a.dtype}")
        return kind, a.shape, a.astype(a.dtype.newbyteorder("<"), copy=False).tobytes()
    if not isinstance(x, torch.Tensor):
        raise TypeError("state entries must be torch tensors or numpy arrays")
    kind = _DTYPES.get(x.dtype)
    if kind is None:
        raise TypeError(f"cannot dump a tensor of dtype {x.dtype}")
    h = x.detach().to("cpu").contiguous()
    if kind == "bf16":
        h = h.view(torch.int16)
    return kind, tuple(h.shape), h.numpy().astype(_NP[kind] if kind != "bf16" else np.int16).tobytes()


def save(path: str, tensors: dict, meta: dict) -> None:
    """Write every non-None entry of `tensors` as `<name>.bin` and `state.json` with `meta`."""
    os.makedirs(path, exist_ok=True)
    index = {}
    for name, x in tensors.items():
        if x is None:
            continue
        if not name.isidentifier():
            raise ValueError(f"bad tensor name {name!r}")
        kind, shape, raw = _host_bytes(x)
        with open(os.path.join(path, name + ".bin"), "wb") as f:
            f.write(raw)
        index[name] = {"dtype": kind, "shape": list(shape)}
    with open(os.path.join(path, "state.json"), "w") as f:
        json.dump({"format": _FORMAT, "tensors": index, "meta": meta}, f, indent=1, sort_keys=True)


def load(path: str, device="cuda") -> tuple[dict, dict]:
    """(tensors, meta) from a directory written by save(); tensors are torch tensors on `device`."""
    with open(os.path.join(path, "state.json")) as f:
        doc = json.load(f)
    if doc.get("format") != _FORMAT:
        raise ValueError(f"unknown state format {doc.get('format')!r}")
    out = {}
    for name, e in doc["tensors"].items():
        kind, shape = e["dtype"], tuple(e["shape"])
        n = int(np.prod(shape, dtype=np.int64))
        np_dtype = np.dtype(_NP[kind]).newbyteorder("<")
        raw = np.fromfile(os.path.join(path, name + ".bin"), dtype=np_dtype)
        if raw.size != n:
            raise ValueError(f"{name}.bin holds {raw.size} elements, state.json says {n}")
        a = raw.astype(np_dtype.newbyteorder("="), copy=False).reshape(shape)
        if kind == "bf16":
            t = torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
        else:
            t = torch.from_numpy(a.copy())
        out[name] = t.to(device)
    return out, doc["meta"]


def cache_state(cache) -> tuple[dict, dict]:
    """(tensors, meta) describing a BoundedKVCache or a PagedKVCache."""
    from .cache import BoundedKVCache, PagedKVCache
    if isinstance(cache, BoundedKVCache):
        meta = dict(kind="flat", B=cache.B, Hq=cache.Hq, Hkv=cache.Hkv, d=cache.d, cap=cache.cap, M=cache.M,
                    num_splits=cache.num_splits, split_len=cache.split_len, with_beta=cache.log_beta is not None)
        t = dict(k=cache.k, v=cache.v, log_beta=cache.log_beta, pos=cache.pos, len=cache.len)
        return t, meta
    if isinstance(cache, PagedKVCache):
        p = cache.pool
        meta = dict(kind="paged", B=cache.B, Hq=cache.Hq, Hkv=cache.Hkv, d=cache.d, M=cache.M,
                    max_pages=p.max_pages, num_pages=p.num_pages, num_splits=cache.num_splits,
                    split_len=cache.split_len, with_beta=p.log_beta_pages is not None)
        t = dict(k_pages=p.k_pages, v_pages=p.v_pages, log_beta_pages=p.log_beta_pages, pos_pages=p.pos_pages,
                 table=p.table, len=p.len, free_pages=p.free_pages, free_count=p.free_count)
        return t, meta
    raise TypeError("cache must be a BoundedKVCache or a PagedKVCache")


_STEP_INPUTS = ("q", "k_new", "v_new", "log_beta_new", "t", "rm_start", "rm_len")


def dump_step(path: str, cache, inputs: dict, extra_meta: dict | None = None) -> None:
    """Dump `cache` as it is now (before the step) and the step's `inputs` (q, k_new, v_new,
    log_beta_new, t; rm_start / rm_len for a compaction after the attention) under `path`."""
    tensors, meta = cache_state(cache)
    bad = set(inputs) - set(_STEP_INPUTS)
    if bad:
        raise ValueError(f"unknown step inputs {sorted(bad)}")
    clash = set(tensors) & {"in_" + k for k in inputs}
    assert not clash
    tensors = dict(tensors)
    tensors.update({"in_" + k: v for k, v in inputs.items() if v is not None})
    meta = dict(meta)
    if extra_meta:
        meta["extra"] = extra_meta
    save(path, tensors, meta)


def cache_from_state(tensors: dict, meta: dict, device="cuda"):
    """A cache with the sizes of `meta` holding the dumped tensors."""
    from .cache import BoundedKVCache, PagedKVCache
    if meta["kind"] == "flat":
        c = BoundedKVCache(meta["B"], meta["Hq"], meta["Hkv"], meta["d"], meta["cap"], meta["M"],
                           num_splits=meta["num_splits"], split_len=meta["split_len"],
                           with_beta=meta["with_beta"], device=device)
        dst = dict(k=c.k, v=c.v, log_beta=c.log_beta, pos=c.pos, len=c.len)
    elif meta["kind"] == "paged":
        c = PagedKVCache(meta["B"], meta["Hq"], meta["Hkv"], meta["d"], meta["max_pages"], meta["num_pages"],
                         meta["M"], num_splits=meta["num_splits"], split_len=meta["split_len"],
                         with_beta=meta["with_beta"], device=device)
        p = c.pool
        dst = dict(k_pages=p.k_pages, v_pages=p.v_pages, log_beta_pages=p.log_beta_pages, pos_pages=p.pos_pages,
                   table=p.table, len=p.len, free_pages=p.free_pages, free_count=p.free_count)
    else:
        raise ValueError(f"unknown cache kind {meta['kind']!r}")
    for name, d in dst.items():
        if d is None:
            continue
        s = tensors[name]
        if s.shape != d.shape or s.dtype != d.dtype:
            raise ValueError(f"{name}: dumped {tuple(s.shape)} {s.dtype}, cache wants {tuple(d.shape)} {d.dtype}")
        d.copy_(s)
    return c


def load_step(path: str, device="cuda"):
    """(cache, inputs, meta) from a directory written by dump_step()."""
    tensors, meta = load(path, device)
    inputs = {k[3:]: v for k, v in tensors.items() if k.startswith("in_")}
    return cache_from_state(tensors, meta, device), inputs, meta


def replay_step(cache, inputs: dict, use_beta: bool = True):
    """Run the dumped step: insertion (with budget enforcement), attention, then the compaction if
    the inputs hold one. Returns (o [B, Hq, d] f32, lse [B, Hq] f32)."""
    q = inputs["q"]
    B, Hq, d = q.shape
    o = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    cache.insert(inputs["k_new"], inputs["v_new"], inputs.get("log_beta_new"), inputs["t"])
    cache.attend(q, inputs["t"], o, lse, use_beta=use_beta)
    if "rm_start" in inputs:
        cache.compact(inputs["rm_start"], inputs["rm_len"])
    return o, lse
