"""CPU oracle for the memory-bounded KV decode path (ctypes wrapper of kvb_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline leg use it; the library never imports, links or runs it. It shares
no code with the CUDA path. Every function takes host numpy arrays (bf16 as
uint16 bit patterns) and returns float64 results.

Parity status (what pins each function, see tests/test_oracle_*.py):
  decode_attn      pinned: library SDPA in float64 (plain and with the
                   retention bias as an additive mask), closed forms,
                   split/merge identity, GQA isolation
  merge_states     pinned: closed form in the Z domain, identity element,
                   commutativity/associativity, merge of blocks == SDPA
  evict_insert     pinned: brute-force minimum of beta^(t-i) in double,
                   FIFO under constant beta, len = min(M, t+1), untouched slots
  compact_blocks   pinned: numpy.delete on the slot axis, attention after
                   compaction == masked SDPA over the old cache
  asm_lookup_merge pinned: sklearn cosine_similarity argmax, exact-match
                   retrieval, merged state == SDPA over prefix + self
  asm_build.asm_aggregate, asm_build.asm_kmeans (numpy, float64)
                   pinned: single members, the two-state Z-domain formula, the
                   pinned n-way merge, chunked prefix build == SDPA over the
                   whole prefix, closed-form means, separated groups recovered
                   by the clustering, objective never decreasing
  decode_steps_threads (parallel driver of evict_insert + decode_attn)
                   pinned: bit-identical to the serial functions called step by
                   step over the whole batch (victims, cache bytes, o, lse)
  asm_hier_lookup_merge
                   pinned: m = C over a partition == sklearn cosine_similarity
                   argmax; constructed indexes with known answers (best
                   centroid outside the selected clusters, coarse ties,
                   empty clusters); merge as asm_lookup_merge
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvb_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
_D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile kvb_oracle.cpp with g++ (IEEE semantics: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-pthread", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_decode_attn.argtypes = [_P, _L, _L, _P, _P, _L, _L, _P, _P, _L, _L, _P, _P,
                                           _I, _I, _I, _I, _I, _D, _I, _I, _P, _P, _P, _P]
        lib.oracle_merge_states.argtypes = [_P, _P, _L, _L, _L, _L, _I, _I, _I, _P, _P]
        lib.oracle_evict_insert.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]
        lib.oracle_compact_blocks.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I]
        lib.oracle_asm_cosines.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P]
        lib.oracle_asm_lookup_merge.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]
        lib.oracle_asm_hier_lookup_merge.argtypes = [_P] * 9 + [_I] * 6 + [_P] * 4
        lib.oracle_decode_steps_threads.argtypes = [_P] * 10 + [_I] * 8 + [_P] * 3
        for f in (lib.oracle_decode_attn, lib.oracle_merge_states, lib.oracle_evict_insert,
                  lib.oracle_compact_blocks, lib.oracle_asm_cosines, lib.oracle_asm_lookup_merge,
                  lib.oracle_asm_hier_lookup_merge, lib.oracle_decode_steps_threads):
            f.restype = _I
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != 0:
        raise OracleError(f"{what}: status {status}")


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def decode_attn(q, k, v, log_beta, pos, len_, t, *, scale=0.0, num_splits=1, split_len=0,
                want_parts=False, kv_batch_stride=None, meta_batch_stride=None):
    """Retention-gated GQA decode attention state per (b, h).

    q [B, Hq, d] uint16; k, v [Bk, Hkv, cap, d] uint16 with Bk == B, or Bk == 1 and
    kv_batch_stride=0 (one cache shared by every row); log_beta (nullable) and pos
    [Bk, Hkv, cap]; len [B, Hkv]; t [B] (nullable when log_beta is None).
    Returns (o [B, Hq, d], lse [B, Hq]) and, with want_parts, (o_part [B, Hq, S, d],
    lse_part [B, Hq, S]) as float64. Raises OracleError on status 3 (bad length).
    """
    lib = _load()
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    log_beta = _c(log_beta, np.float32)
    pos = _c(pos, np.int32)
    len_ = _c(len_, np.int32)
    t = _c(t, np.int32)
    B, Hq, d = q.shape
    _, Hkv, cap, _ = k.shape
    kv_sb = Hkv * cap * d if kv_batch_stride is None else kv_batch_stride
    m_sb = Hkv * cap if meta_batch_stride is None else meta_batch_stride
    S = int(num_splits)
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    op = np.zeros((B, Hq, S, d), np.float64) if want_parts else None
    lp = np.zeros((B, Hq, S), np.float64) if want_parts else None
    st = lib.oracle_decode_attn(_ptr(q), Hq * d, d, _ptr(k), _ptr(v), kv_sb, cap * d,
                                _ptr(log_beta), _ptr(pos), m_sb, cap, _ptr(len_), _ptr(t),
                                B, Hq, Hkv, d, cap, float(scale), S, int(split_len),
                                _ptr(o), _ptr(lse), _ptr(op), _ptr(lp))
    _check(st, "oracle_decode_attn")
    return (o, lse, op, lp) if want_parts else (o, lse)


def merge_states(o_in, lse_in):
    """Merge n states per row: o_in [n, R, d], lse_in [n, R] -> (o [R, d], lse [R]) in float64."""
    lib = _load()
    o_in = _c(o_in, np.float64)
    lse_in = _c(lse_in, np.float64)
    n, R, d = o_in.shape
    o = np.zeros((R, d), np.float64)
    lse = np.zeros((R,), np.float64)
    _check(lib.oracle_merge_states(_ptr(o_in), _ptr(lse_in), R * d, d, R, 1, n, R, d,
                                   _ptr(o), _ptr(lse)), "oracle_merge_states")
    return o, lse


def evict_insert(cache: dict, k_new, v_new, log_beta_new, t, M: int):
    """Budget enforcement + insertion on a host cache dict {k, v, log_beta, pos, len} (in place).

    Returns victim [B, Hkv] int32 (-1 = appended or inactive)."""
    lib = _load()
    k, v, lb, pos, ln = cache["k"], cache["v"], cache.get("log_beta"), cache["pos"], cache["len"]
    for a in (k, v, pos, ln) + ((lb,) if lb is not None else ()):
        assert a.flags.c_contiguous
    B, Hkv, cap, d = k.shape
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    log_beta_new = _c(log_beta_new, np.float32)
    t = _c(t, np.int32)
    victim = np.zeros((B, Hkv), np.int32)
    _check(lib.oracle_evict_insert(_ptr(k), _ptr(v), _ptr(lb), _ptr(pos), _ptr(ln), _ptr(k_new),
                                   _ptr(v_new), _ptr(log_beta_new), _ptr(t), B, Hkv, d, cap, int(M),
                                   _ptr(victim)), "oracle_evict_insert")
    return victim


def decode_steps_threads(cache: dict, q, k_new, v_new, log_beta_new, t, M: int, nthreads: int = 0):
    """`steps` decode steps (evict_insert, then decode_attn with one split) on a host cache dict,
    in place, with the (sequence, kv head) units spread over `nthreads` threads (0 = all cores).

    q [steps, B, Hq, d] or None (no attention); k_new, v_new [steps, B, Hkv, d] or None;
    log_beta_new [steps, B, Hkv]; t [steps, B]. Each thread runs the serial functions on one
    unit's slice, so the results equal evict_insert + decode_attn called step by step.
    Returns (victim [steps, B, Hkv], o [B, Hq, d], lse [B, Hq]) -- o, lse of the last step,
    None when q is None."""
    lib = _load()
    k, v, lb, pos, ln = cache["k"], cache["v"], cache.get("log_beta"), cache["pos"], cache["len"]
    for a in (k, v, pos, ln) + ((lb,) if lb is not None else ()):
        assert a.flags.c_contiguous
    B, Hkv, cap, d = k.shape
    t = _c(t, np.int32)
    steps = t.shape[0]
    q = _c(q, np.uint16)
    Hq = q.shape[2] if q is not None else Hkv
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    log_beta_new = _c(log_beta_new, np.float32)
    victim = np.zeros((steps, B, Hkv), np.int32)
    o = np.zeros((B, Hq, d), np.float64) if q is not None else None
    lse = np.zeros((B, Hq), np.float64) if q is not None else None
    _check(lib.oracle_decode_steps_threads(_ptr(k), _ptr(v), _ptr(lb), _ptr(pos), _ptr(ln), _ptr(q), _ptr(k_new),
                                           _ptr(v_new), _ptr(log_beta_new), _ptr(t), steps, B, Hq, Hkv, d, cap,
                                           int(M), int(nthreads), _ptr(victim), _ptr(o), _ptr(lse)),
           "oracle_decode_steps_threads")
    return victim, o, lse


def compact_blocks(cache: dict, rm_start, rm_len):
    """In-place removal of slot range [rm_start[b], +rm_len[b]) from every head of sequence b."""
    lib = _load()
    k, v, lb, pos, ln = cache["k"], cache["v"], cache.get("log_beta"), cache["pos"], cache["len"]
    B, Hkv, cap, d = k.shape
    rm_start = _c(rm_start, np.int32)
    rm_len = _c(rm_len, np.int32)
    _check(lib.oracle_compact_blocks(_ptr(k), _ptr(v), _ptr(pos), _ptr(lb), _ptr(ln), _ptr(rm_start),
                                     _ptr(rm_len), B, Hkv, d, cap), "oracle_compact_blocks")


def asm_cosines(q, qbar, n: int, h: int):
    lib = _load()
    q = _c(q, np.uint16)
    qbar = _c(qbar, np.float32)
    N, H, d = q.shape
    K = qbar.shape[1]
    out = np.zeros(K, np.float64)
    _check(lib.oracle_asm_cosines(_ptr(q), _ptr(qbar), N, H, K, d, int(n), int(h), _ptr(out)),
           "oracle_asm_cosines")
    return out


def asm_lookup_merge(q, qbar, abar, log_zbar, o_self, lse_self):
    """Returns (idx [N, H] int32, o [N, H, d] float64, lse [N, H] float64)."""
    lib = _load()
    q = _c(q, np.uint16)
    qbar = _c(qbar, np.float32)
    abar = _c(abar, np.uint16)
    log_zbar = _c(log_zbar, np.float32)
    o_self = _c(o_self, np.float32)
    lse_self = _c(lse_self, np.float32)
    N, H, d = q.shape
    K = qbar.shape[1]
    idx = np.zeros((N, H), np.int32)
    o = np.zeros((N, H, d), np.float64)
    lse = np.zeros((N, H), np.float64)
    _check(lib.oracle_asm_lookup_merge(_ptr(q), _ptr(qbar), _ptr(abar), _ptr(log_zbar), _ptr(o_self),
                                       _ptr(lse_self), N, H, K, d, _ptr(idx), _ptr(o), _ptr(lse)),
           "oracle_asm_lookup_merge")
    return idx, o, lse


def asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, log_zbar, o_self, lse_self, m: int):
    """Two-level lookup. Returns (sel [N, H, m] int32, idx [N, H] int32, o [N, H, d] float64,
    lse [N, H] float64); idx = -1 where the selected clusters hold no member."""
    lib = _load()
    q = _c(q, np.uint16)
    qhat = _c(qhat, np.float32)
    offsets = _c(offsets, np.int32)
    members = _c(members, np.int32)
    qbar = _c(qbar, np.float32)
    abar = _c(abar, np.uint16)
    log_zbar = _c(log_zbar, np.float32)
    o_self = _c(o_self, np.float32)
    lse_self = _c(lse_self, np.float32)
    N, H, d = q.shape
    K = qbar.shape[1]
    C = qhat.shape[1]
    sel = np.zeros((N, H, m), np.int32)
    idx = np.zeros((N, H), np.int32)
    o = np.zeros((N, H, d), np.float64)
    lse = np.zeros((N, H), np.float64)
    _check(lib.oracle_asm_hier_lookup_merge(_ptr(q), _ptr(qhat), _ptr(offsets), _ptr(members), _ptr(qbar),
                                            _ptr(abar), _ptr(log_zbar), _ptr(o_self), _ptr(lse_self), N, H, K,
                                            C, int(m), d, _ptr(sel), _ptr(idx), _ptr(o), _ptr(lse)),
           "oracle_asm_hier_lookup_merge")
    return sel, idx, o, lse
