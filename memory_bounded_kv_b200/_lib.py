"""ctypes declarations of the C ABI in include/kvb.h (libkvb.so, built in-tree)."""
from __future__ import annotations

import ctypes
import os

from . import _build

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

# symbols include/kvb.h declares (kept in sync by tests/test_abi.py)
EXPORTS = (
    "kvb_decode_attn", "kvb_decode_attn_noalloc", "kvb_decode_step", "kvb_merge_states", "kvb_evict_insert",
    "kvb_compact_blocks", "kvb_asm_workspace_bytes", "kvb_asm_lookup_merge", "kvb_asm_hier_workspace_bytes",
    "kvb_asm_hier_lookup_merge", "kvb_asm_aggregate_workspace_bytes", "kvb_asm_aggregate",
    "kvb_asm_entries_bf16", "kvb_asm_index_workspace_bytes", "kvb_asm_index_csr",
    "kvb_asm_lookup_merge_grouped", "kvb_asm_aggregate_grouped",
    "kvb_get_error", "kvb_status_str",
    "kvb_abi_version", "kvb_test_withhold_next_decode",
    "kvb_paged_reset", "kvb_paged_evict_insert", "kvb_paged_decode_attn", "kvb_paged_compact_blocks",
    "kvb_asm_planes_bytes", "kvb_asm_prepare", "kvb_asm_lookup_merge_planes",
)

KVB_OK, KVB_EINVAL, KVB_ECUDA, KVB_EDEVICE = 0, 1, 2, 3
KVB_OUT_F32, KVB_OUT_BF16 = 0, 1
DERR_LEN, DERR_SPLIT, DERR_RANGE, DERR_TIMEOUT, DERR_PAGES, DERR_STEP = 1, 2, 4, 8, 16, 32
NOALLOC_SCRATCH_BYTES = 16 << 20   # KVB_NOALLOC_SCRATCH_BYTES


class AttnArgs(ctypes.Structure):
    """Mirror of struct kvb_attn_args."""
    _fields_ = [
        ("q", _P), ("q_stride_b", _I64), ("q_stride_h", _I64),
        ("k", _P), ("v", _P), ("kv_stride_b", _I64), ("kv_stride_h", _I64),
        ("log_beta", _P), ("pos", _P), ("meta_stride_b", _I64), ("meta_stride_h", _I64),
        ("len", _P), ("t", _P),
        ("B", _I32), ("Hq", _I32), ("Hkv", _I32), ("d", _I32), ("cap", _I32),
        ("scale", ctypes.c_float),
        ("num_splits", _I32), ("split_len", _I32),
        ("o_part", _P), ("lse_part", _P), ("counters", _P),
        ("o", _P), ("o_dtype", _I32), ("lse", _P),
        ("evict_cand", _P),
    ]

EVICT_CAND_BYTES = 16   # sizeof(kvb_evict_cand)
PAGE_SLOTS = 64         # KVB_PAGE_SLOTS


class PagedCacheArgs(ctypes.Structure):
    """Mirror of struct kvb_paged_cache."""
    _fields_ = [
        ("k_pages", _P), ("v_pages", _P), ("log_beta_pages", _P), ("pos_pages", _P),
        ("table", _P), ("len", _P), ("free_pages", _P), ("free_count", _P),
        ("B", _I32), ("Hkv", _I32), ("d", _I32), ("max_pages", _I32), ("num_pages", _I32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkvb.so, building it first if it is missing or older than its sources."""
    global _lib
    if _lib is None:
        path = _build.SO
        if _build.stale():
            try:
                path = _build.build()
            except Exception as e:  # no nvcc and no prebuilt library: the CUDA path is unavailable
                raise RuntimeError(f"libkvb.so is missing and could not be built: {e}") from e
        if not os.path.exists(path):
            raise RuntimeError(f"libkvb.so not found at {path}")
        L = ctypes.CDLL(path)
        L.kvb_decode_attn.argtypes = [ctypes.POINTER(AttnArgs), _P]
        L.kvb_decode_attn_noalloc.argtypes = [ctypes.POINTER(AttnArgs), _P]
        L.kvb_decode_step.argtypes = [ctypes.POINTER(AttnArgs), _P, _P, _P, _I32, _P, _P, _P]
        L.kvb_merge_states.argtypes = [_P, _P, _I64, _I64, _I64, _I64, _I32, _I32, _I32, _P, _P, _P]
        L.kvb_evict_insert.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P, _P,
                                       _I32, _P]
        L.kvb_compact_blocks.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _P]
        L.kvb_asm_workspace_bytes.argtypes = [_I32, _I32, _I32]
        L.kvb_asm_workspace_bytes.restype = _SZ
        L.kvb_asm_lookup_merge.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _SZ, _P]
        L.kvb_asm_hier_workspace_bytes.argtypes = [_I32, _I32, _I32]
        L.kvb_asm_hier_workspace_bytes.restype = _SZ
        L.kvb_asm_hier_lookup_merge.argtypes = [_P] * 9 + [_I32] * 6 + [_P, _P, _P, _P, _SZ, _P]
        L.kvb_asm_aggregate_workspace_bytes.argtypes = [_I32, _I32]
        L.kvb_asm_aggregate_workspace_bytes.restype = _SZ
        L.kvb_asm_aggregate.argtypes = [_P] * 4 + [_I32] * 5 + [_P] * 5 + [_SZ, _P]
        L.kvb_asm_entries_bf16.argtypes = [_P, _I32, _I32, _I32, _P, _P]
        L.kvb_asm_index_workspace_bytes.argtypes = [_I32, _I32]
        L.kvb_asm_index_workspace_bytes.restype = _SZ
        L.kvb_asm_index_csr.argtypes = [_P, _I32, _I32, _I32, _P, _P, _P, _SZ, _P]
        L.kvb_asm_lookup_merge_grouped.argtypes = [_P] * 6 + [_I32] * 5 + [_P] * 4 + [_SZ, _P]
        L.kvb_asm_aggregate_grouped.argtypes = [_P] * 4 + [_I32] * 6 + [_P] * 5 + [_SZ, _P]
        L.kvb_get_error.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
        L.kvb_status_str.argtypes = [_I32]
        L.kvb_status_str.restype = ctypes.c_char_p
        L.kvb_abi_version.argtypes = []
        L.kvb_test_withhold_next_decode.argtypes = [ctypes.c_uint64]
        _PC = ctypes.POINTER(PagedCacheArgs)
        L.kvb_paged_reset.argtypes = [_PC, _P]
        L.kvb_paged_evict_insert.argtypes = [_PC, _P, _P, _P, _P, _I32, _P, _P, _I32, _P]
        L.kvb_paged_decode_attn.argtypes = [_PC, _P, _P, _I32, ctypes.c_float, _I32, _I32, _P, _P, _P, _I32, _P, _P,
                                            _P]
        L.kvb_paged_compact_blocks.argtypes = [_PC, _P, _P, _P]
        L.kvb_asm_planes_bytes.argtypes = [_I32, _I32]
        L.kvb_asm_planes_bytes.restype = _SZ
        L.kvb_asm_prepare.argtypes = [_P, _I32, _I32, _I32, _P, _SZ, _P]
        L.kvb_asm_lookup_merge_planes.argtypes = [_P, _P, _SZ, _P, _P, _P, _P] + [_I32] * 5 + [_P] * 4 + [_SZ, _P]
        for f in ("kvb_decode_attn", "kvb_decode_attn_noalloc", "kvb_decode_step", "kvb_merge_states", "kvb_evict_insert", "kvb_compact_blocks",
                  "kvb_asm_lookup_merge", "kvb_asm_hier_lookup_merge", "kvb_asm_aggregate",
                  "kvb_asm_entries_bf16", "kvb_asm_index_csr", "kvb_asm_lookup_merge_grouped",
                  "kvb_asm_aggregate_grouped", "kvb_get_error",
                  "kvb_abi_version", "kvb_test_withhold_next_decode", "kvb_paged_reset",
                  "kvb_paged_evict_insert", "kvb_paged_decode_attn", "kvb_paged_compact_blocks",
                  "kvb_asm_prepare", "kvb_asm_lookup_merge_planes"):
            getattr(L, f).restype = _I32
        _lib = L
    return _lib
