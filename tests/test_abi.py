"""The C-ABI library builds for sm_100a, loads, and exports every entry point
include/kvb.h declares; host-side argument checks reject bad arguments before
any launch (these calls need no GPU: nothing reaches the device)."""
import ctypes
import os
import re

import pytest

from memory_bounded_kv_b200 import _lib, _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvb.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvb_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = _lib.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {_build.SO}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_attn_args_struct_matches_header():
    src = open(HEADER).read()
    body = re.search(r"typedef struct kvb_attn_args \{(.*?)\} kvb_attn_args;", src, re.S).group(1)
    names = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        decl = re.sub(r"^(const\s+)?\w+\s*\**\s*", "", decl)
        names += [n.strip().lstrip("*") for n in decl.split(",")]
    assert names == [f[0] for f in _lib.AttnArgs._fields_]


def test_status_strings_and_version():
    L = _lib.lib()
    assert L.kvb_abi_version() == 7
    assert L.kvb_status_str(0) == b"ok"
    assert L.kvb_status_str(1) == b"invalid argument"


def _args(**kw):
    fake = 1 << 20  # a 16-byte aligned non-null value; the host checks never dereference it
    a = dict(q=fake, q_stride_b=32 * 128, q_stride_h=128, k=fake, v=fake, kv_stride_b=8 * 64 * 128,
             kv_stride_h=64 * 128, log_beta=None, pos=None, meta_stride_b=0, meta_stride_h=0, len=fake, t=None,
             B=2, Hq=32, Hkv=8, d=128, cap=64, scale=0.0, num_splits=1, split_len=0, o_part=None, lse_part=None,
             counters=None, o=fake, o_dtype=0, lse=None)
    a.update(kw)
    return _lib.AttnArgs(**a)


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(Hq=12), dict(Hq=48, Hkv=3), dict(num_splits=0), dict(num_splits=2),
    dict(q=(1 << 20) + 2), dict(kv_stride_h=100), dict(log_beta=1 << 20), dict(o_dtype=5),
    dict(scale=float("nan")), dict(B=0), dict(split_len=-1), dict(q=None),
    dict(o=(1 << 20) + 4),                                                         # outputs 16-byte aligned
    dict(num_splits=2, split_len=32, o_part=(1 << 20) + 8, lse_part=1 << 20),
])
def test_decode_attn_rejects_bad_arguments_on_the_host(bad):
    L = _lib.lib()
    assert L.kvb_decode_attn(ctypes.byref(_args(**bad)), None) == _lib.KVB_EINVAL


def test_other_entry_points_reject_bad_arguments_on_the_host():
    L = _lib.lib()
    f = ctypes.c_void_p(1 << 20)
    assert L.kvb_evict_insert(f, f, None, f, f, f, f, None, f, 1, 1, 128, 64, 65, None, None, 0, None) == _lib.KVB_EINVAL
    assert L.kvb_evict_insert(f, f, None, f, f, f, None, None, f, 1, 1, 128, 64, 8, None, None, 0, None) == _lib.KVB_EINVAL
    # candidates: count out of range, misaligned buffer
    assert L.kvb_evict_insert(f, f, None, f, f, f, f, None, f, 1, 1, 128, 64, 8, None, f, 0, None) == _lib.KVB_EINVAL
    assert L.kvb_evict_insert(f, f, None, f, f, f, f, None, f, 1, 1, 128, 64, 8, None,
                              ctypes.c_void_p((1 << 20) + 8), 2, None) == _lib.KVB_EINVAL
    assert L.kvb_compact_blocks(f, f, f, None, f, f, f, 1, 1, 12, 64, None) == _lib.KVB_EINVAL
    assert L.kvb_merge_states(f, f, 1, 1, 1, 1, 0, 4, 8, f, None, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_lookup_merge(f, f, f, f, f, f, 4, 2, 16, 64, None, f, None, f, 1 << 20, None) == _lib.KVB_EINVAL
    # two-level lookup: C, m out of range, short workspace, misaligned members
    assert L.kvb_asm_hier_lookup_merge(f, f, f, f, f, f, f, f, f, 1, 2, 64, 0, 4, 128, None, f, None, f, 1 << 20,
                                       None) == _lib.KVB_EINVAL
    assert L.kvb_asm_hier_lookup_merge(f, f, f, f, f, f, f, f, f, 1, 2, 64, 1025, 4, 128, None, f, None, f, 1 << 20,
                                       None) == _lib.KVB_EINVAL
    assert L.kvb_asm_hier_lookup_merge(f, f, f, f, f, f, f, f, f, 1, 2, 64, 8, 65, 128, None, f, None, f, 1 << 20,
                                       None) == _lib.KVB_EINVAL
    assert L.kvb_asm_hier_workspace_bytes(3, 2, 16) == 3 * 2 * 16 * 12
    assert L.kvb_asm_hier_lookup_merge(f, f, f, f, f, f, f, f, f, 3, 2, 64, 8, 16, 128, None, f, None, f,
                                       3 * 2 * 16 * 12 - 1, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_hier_lookup_merge(f, f, f, ctypes.c_void_p((1 << 20) + 2), f, f, f, f, f, 1, 2, 64, 8, 4, 128,
                                       None, f, None, f, 1 << 20, None) == _lib.KVB_EINVAL
    # aggregation: a without lse, d != 128, short workspace; assignment-only lookup without idx
    assert L.kvb_asm_aggregate(f, f, None, f, 10, 2, 8, 128, 0, f, f, f, None, f, 1 << 24, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_aggregate(f, None, None, f, 10, 2, 8, 64, 0, f, None, None, None, f, 1 << 24,
                               None) == _lib.KVB_EINVAL
    assert L.kvb_asm_aggregate_workspace_bytes(2, 8) == 2 * 8 * 12 + 2 * 2 * 8 * 128 * 4
    assert L.kvb_asm_aggregate(f, None, None, f, 10, 2, 8, 128, 0, f, None, None, None, f,
                               2 * 8 * 12 + 2 * 2 * 8 * 128 * 4 - 1, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_lookup_merge(f, f, None, None, None, None, 4, 2, 16, 128, None, None, None, f, 1 << 20,
                                  None) == _lib.KVB_EINVAL
    # index: d != 128, misaligned output, C out of range, short workspace
    assert L.kvb_asm_entries_bf16(f, 2, 8, 64, f, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_entries_bf16(f, 2, 8, 128, ctypes.c_void_p((1 << 20) + 8), None) == _lib.KVB_EINVAL
    assert L.kvb_asm_index_csr(f, 100, 2, 0, f, f, f, 1 << 20, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_index_workspace_bytes(2, 7) == 2 * 7 * 4
    assert L.kvb_asm_index_csr(f, 100, 2, 7, f, f, f, 2 * 7 * 4 - 1, None) == _lib.KVB_EINVAL
    # grouped tables must divide the heads
    assert L.kvb_asm_lookup_merge_grouped(f, f, f, f, f, f, 4, 6, 4, 16, 128, None, f, None, f, 1 << 20,
                                          None) == _lib.KVB_EINVAL
    assert L.kvb_asm_aggregate_grouped(f, None, None, f, 10, 6, 0, 8, 128, 0, f, None, None, None, f, 1 << 24,
                                       None) == _lib.KVB_EINVAL
    ws = L.kvb_asm_workspace_bytes(256, 32, 4096)
    assert ws == 32 * 256 * 32 * 8   # 32 ranges of 128 centroids, one 8-byte key per (range, query, head)
    assert L.kvb_asm_lookup_merge(f, f, f, f, f, f, 256, 32, 4096, 128, None, f, None, f, ws - 1, None) == _lib.KVB_EINVAL


def test_paged_and_planes_entry_points_reject_bad_arguments_on_the_host():
    L = _lib.lib()
    f = 1 << 20
    pc = _lib.PagedCacheArgs(k_pages=f, v_pages=f, log_beta_pages=None, pos_pages=f, table=f, len=f, free_pages=f,
                             free_count=f, B=2, Hkv=2, d=128, max_pages=4, num_pages=16)
    p = ctypes.c_void_p(f)
    # several splits must start on pages: split_len a positive multiple of 64
    assert L.kvb_paged_decode_attn(ctypes.byref(pc), p, p, 8, 0.0, 2, 0, p, p, p, 0, None, None, None) == _lib.KVB_EINVAL
    assert L.kvb_paged_decode_attn(ctypes.byref(pc), p, p, 8, 0.0, 2, 100, p, p, p, 0, None, None, None) == _lib.KVB_EINVAL
    assert L.kvb_paged_decode_attn(ctypes.byref(pc), p, p, 12, 0.0, 1, 0, None, None, p, 0, None, None, None) == _lib.KVB_EINVAL
    # budget above the capacity of the table
    assert L.kvb_paged_evict_insert(ctypes.byref(pc), p, p, None, p, 4 * 64 + 1, None, None, 0, None) == _lib.KVB_EINVAL
    bad = _lib.PagedCacheArgs(k_pages=f + 8, v_pages=f, log_beta_pages=None, pos_pages=f, table=f, len=f,
                              free_pages=f, free_count=f, B=2, Hkv=2, d=128, max_pages=4, num_pages=16)
    assert L.kvb_paged_reset(ctypes.byref(bad), None) == _lib.KVB_EINVAL
    assert L.kvb_paged_compact_blocks(ctypes.byref(pc), None, p, None) == _lib.KVB_EINVAL
    # prepared memory: size of the planes, and refusals
    assert L.kvb_asm_planes_bytes(2, 100) == 2 * 2 * 3 * 2 * 64 * 128
    assert L.kvb_asm_prepare(p, 2, 100, 64, p, 1 << 30, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_prepare(p, 2, 100, 128, p, 1000, None) == _lib.KVB_EINVAL
    assert L.kvb_asm_lookup_merge_planes(p, p, 1000, p, p, p, p, 4, 2, 2, 100, 128, None, p, None, p, 1 << 20,
                                         None) == _lib.KVB_EINVAL
