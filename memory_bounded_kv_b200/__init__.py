"""memory_bounded_kv_b200: decode-step attention over a memory-bounded KV cache on B200.

Python binding of libkvb (include/kvb.h). Each function has the name of a C
entry point and only marshals arguments: it checks dtypes, devices and layouts
of torch tensors, passes their device pointers and strides, and raises
KvbError when the library returns a non-OK status (kvb_asm_lookup_merge and
kvb_asm_aggregate call the _grouped entry points, with the table count taken
from qbar's first dimension). Every step of the path runs in the library's
CUDA kernels; there is no other implementation.

Modules: cache (BoundedKVCache: the decode step of one layer), asm_build (the
memory's offline build: clustering, aggregation, two-level index), synth
(seeded synthetic workloads).

bf16 tensors are torch.bfloat16. Calls run on `stream` (default: torch's
current stream) and are asynchronous.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

__all__ = [
    "KvbError", "kvb_decode_attn", "kvb_decode_attn_noalloc", "kvb_decode_step", "kvb_merge_states", "kvb_evict_insert", "kvb_compact_blocks",
    "kvb_asm_workspace_bytes", "kvb_asm_lookup_merge", "kvb_asm_hier_workspace_bytes",
    "kvb_asm_hier_lookup_merge", "kvb_asm_aggregate_workspace_bytes", "kvb_asm_aggregate",
    "kvb_asm_entries_bf16", "kvb_asm_index_workspace_bytes", "kvb_asm_index_csr",
    "kvb_asm_lookup_merge_grouped", "kvb_asm_aggregate_grouped",
    "kvb_get_error", "kvb_abi_version", "kvb_test_withhold_next_decode",
    "decode_workspace", "evict_candidates",
    "PagedPool", "kvb_paged_reset", "kvb_paged_evict_insert", "kvb_paged_decode_attn", "kvb_paged_compact_blocks",
    "kvb_asm_planes_bytes", "kvb_asm_prepare", "kvb_asm_lookup_merge_planes",
]


class KvbError(RuntimeError):
    def __init__(self, status: int, where: str, bits: int = 0):
        msg = _lib.lib().kvb_status_str(status).decode()
        super().__init__(f"{where}: {msg} (status {status}{', device error bits %#x' % bits if bits else ''})")
        self.status = status
        self.bits = bits


def _check(status: int, where: str):
    if status != _lib.KVB_OK:
        raise KvbError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t, dtype, name, cuda=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if cuda and not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    return t


def _contig(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(t, shape, name):
    """Raise ValueError unless tensor t (skipped when None) has exactly `shape`. The library
    cannot see buffer sizes, so every tensor is checked here before anything is launched."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _decode_shapes(q, k, v, log_beta, pos, len, t, o, lse, num_splits, o_part=None, lse_part=None):
    """Shapes of every kvb_decode_attn(_noalloc) argument, from q [B, Hq, d] and k [B, Hkv, cap, d]."""
    if q.dim() != 3 or k.dim() != 4:
        raise ValueError("q must be [B, Hq, d] and k, v [B, Hkv, cap, d]")
    B, Hq, d = q.shape
    _, Hkv, cap, _ = k.shape
    _shape(k, (B, Hkv, cap, d), "k")
    _shape(v, (B, Hkv, cap, d), "v")
    _shape(log_beta, (B, Hkv, cap), "log_beta")
    _shape(pos, (B, Hkv, cap), "pos")
    _shape(len, (B, Hkv), "len")
    _shape(t, (B,), "t")
    _shape(o, (B, Hq, d), "o")
    _shape(lse, (B, Hq), "lse")
    if int(num_splits) < 1:
        raise ValueError("num_splits must be >= 1")
    _shape(o_part, (B, Hq, num_splits, d), "o_part")
    _shape(lse_part, (B, Hq, num_splits), "lse_part")
    return B, Hq, Hkv, d, cap


def kvb_abi_version() -> int:
    return int(_lib.lib().kvb_abi_version())


def kvb_test_withhold_next_decode(wait_limit_ns: int) -> None:
    """Testing hook: the next decode-attention call's producers withhold their copies, so its
    bounded waits run out after wait_limit_ns (see kvb_test_withhold_next_decode in kvb.h)."""
    _check(_lib.lib().kvb_test_withhold_next_decode(int(wait_limit_ns)), "kvb_test_withhold_next_decode")


def kvb_get_error(stream=None) -> int:
    """Synchronize `stream`, read and clear the device error word; returns its bits (0 = none)."""
    bits = ctypes.c_uint32(0)
    st = _lib.lib().kvb_get_error(_stream(stream), ctypes.byref(bits))
    if st not in (_lib.KVB_OK, _lib.KVB_EDEVICE):
        raise KvbError(st, "kvb_get_error")
    return int(bits.value)


def evict_candidates(B: int, Hkv: int, num_splits: int, device="cuda"):
    """Buffer of B*Hkv*num_splits kvb_evict_cand records (16 bytes each) as an int64 tensor."""
    return torch.empty(B * Hkv * num_splits * 2, dtype=torch.int64, device=device)


def _cand_ptr(c, records):
    if not isinstance(c, torch.Tensor) or not c.is_cuda or not c.is_contiguous():
        raise TypeError("evict candidates must be a contiguous CUDA tensor")
    if c.numel() * c.element_size() < records * _lib.EVICT_CAND_BYTES:
        raise ValueError("evict candidate buffer too small")
    return c.data_ptr()


def decode_workspace(B: int, Hq: int, d: int, num_splits: int, device="cuda"):
    """(o_part [B, Hq, S, d], lse_part [B, Hq, S]) f32 buffers for kvb_decode_attn with num_splits > 1."""
    o_part = torch.zeros(B, Hq, num_splits, d, dtype=torch.float32, device=device)
    lse_part = torch.zeros(B, Hq, num_splits, dtype=torch.float32, device=device)
    return o_part, lse_part


def kvb_decode_attn(q, k, v, log_beta, pos, len, t, o, lse=None, *, scale: float = 0.0,
                    num_splits: int = 1, split_len: int = 0, o_part=None, lse_part=None,
                    evict_cand=None, stream=None) -> None:
    """Split-K GQA decode attention with retention bias; see kvb_decode_attn in include/kvb.h.

    q [B, Hq, d] bf16; k, v [B, Hkv, cap, d] bf16 (stride(2) == d, stride(3) == 1; an expanded
    view with stride(0) == 0 shares one cache); log_beta [B, Hkv, cap] f32 or None; pos
    [B, Hkv, cap] int32 (same strides as log_beta); len [B, Hkv] int32; t [B] int32 or None;
    o [B, Hq, d] f32 or bf16; lse [B, Hq] f32 or None; o_part [B, Hq, S, d] / lse_part
    [B, Hq, S] from decode_workspace() when num_splits = S > 1; evict_cand: a CUDA tensor of
    >= B*Hkv*num_splits*16 bytes to receive the next position's eviction candidates (see
    evict_candidates()), or None. Every shape is checked before anything is launched.
    """
    a = _attn_args(q, k, v, log_beta, pos, len, t, o, lse, scale, num_splits, split_len, o_part, lse_part,
                   evict_cand)
    _check(_lib.lib().kvb_decode_attn(ctypes.byref(a), _stream(stream)), "kvb_decode_attn")


def kvb_decode_step(q, k, v, log_beta, pos, len, t, o, lse, k_new, v_new, log_beta_new, M: int, cand_in,
                    cand_out, *, victim=None, scale: float = 0.0, num_splits: int = 1, split_len: int = 0,
                    o_part=None, lse_part=None, stream=None) -> None:
    """Budget enforcement, insertion and attention of a full cache in one launch; see
    kvb_decode_step in include/kvb.h. The arguments of kvb_decode_attn, plus k_new, v_new
    [B, Hkv, d] bf16, log_beta_new [B, Hkv] f32 (exactly when log_beta is given), the budget M,
    cand_in (the records the previous attention left, stamped t) and cand_out (the records for
    t + 1; a different buffer), victim [B, Hkv] int32 or None. k, v, log_beta and pos are written.
    """
    if cand_out is None or cand_in is None:
        raise ValueError("cand_in and cand_out are required")
    if q.dim() != 3 or k.dim() != 4:
        raise ValueError("q must be [B, Hq, d] and k, v [B, Hkv, cap, d]")
    B, Hkv, d = int(q.shape[0]), int(k.shape[1]), int(q.shape[2])
    # shapes first (they need no device), then the attention's checks, then dtypes and devices
    _shape(k_new, (B, Hkv, d), "k_new")
    _shape(v_new, (B, Hkv, d), "v_new")
    if (log_beta is None) != (log_beta_new is None):
        raise ValueError("log_beta_new is needed exactly when log_beta is given")
    _shape(log_beta_new, (B, Hkv), "log_beta_new")
    if victim is not None and victim.numel() < B * Hkv:
        raise ValueError("victim must hold B * Hkv entries")
    a = _attn_args(q, k, v, log_beta, pos, len, t, o, lse, scale, num_splits, split_len, o_part, lse_part,
                   cand_out)
    for name, x in (("k_new", k_new), ("v_new", v_new)):
        _need(x, torch.bfloat16, name); _contig(x, name)
    if log_beta_new is not None:
        _need(log_beta_new, torch.float32, "log_beta_new"); _contig(log_beta_new, "log_beta_new")
    if victim is not None:
        _need(victim, torch.int32, "victim"); _contig(victim, "victim")
    cin = _cand_ptr(cand_in, B * Hkv * int(num_splits))
    _check(_lib.lib().kvb_decode_step(ctypes.byref(a), k_new.data_ptr(), v_new.data_ptr(),
                                      None if log_beta_new is None else log_beta_new.data_ptr(), int(M), cin,
                                      None if victim is None else victim.data_ptr(), _stream(stream)),
           "kvb_decode_step")


def _attn_args(q, k, v, log_beta, pos, len, t, o, lse, scale, num_splits, split_len, o_part, lse_part,
               evict_cand):
    """Checks and marshals the arguments of kvb_decode_attn (and kvb_decode_step) into AttnArgs."""
    B, Hq, Hkv, d, cap = _decode_shapes(q, k, v, log_beta, pos, len, t, o, lse, num_splits, o_part, lse_part)
    if num_splits > 1 and (o_part is None or lse_part is None):
        raise ValueError("num_splits > 1 needs o_part and lse_part (decode_workspace())")
    _need(q, torch.bfloat16, "q"); _need(k, torch.bfloat16, "k"); _need(v, torch.bfloat16, "v")
    if q.stride(2) != 1 or k.stride(3) != 1 or k.stride(2) != d or v.stride() != k.stride():
        raise ValueError("q/k/v: innermost dim contiguous, slot stride d, k and v with equal strides")
    _need(len, torch.int32, "len"); _contig(len, "len")
    meta = None   # the tensor whose strides describe log_beta and pos
    if log_beta is not None:
        _need(log_beta, torch.float32, "log_beta")
        _need(pos, torch.int32, "pos")
        if log_beta.stride() != pos.stride() or log_beta.stride(2) != 1:
            raise ValueError("log_beta and pos need equal strides with slot stride 1")
        _need(t, torch.int32, "t")
        meta = log_beta
    elif pos is not None:
        _need(pos, torch.int32, "pos")
        if pos.stride(2) != 1:
            raise ValueError("pos needs slot stride 1")
        meta = pos
    if t is not None:
        _need(t, torch.int32, "t"); _contig(t, "t")
    if o.dtype == torch.float32:
        odt = _lib.KVB_OUT_F32
    elif o.dtype == torch.bfloat16:
        odt = _lib.KVB_OUT_BF16
    else:
        raise TypeError("o must be float32 or bfloat16")
    _contig(o, "o")
    if lse is not None:
        _need(lse, torch.float32, "lse"); _contig(lse, "lse")
    for name, x in (("o_part", o_part), ("lse_part", lse_part)):
        if x is not None:
            _need(x, torch.float32, name); _contig(x, name)
    a = _lib.AttnArgs(
        q=q.data_ptr(), q_stride_b=q.stride(0), q_stride_h=q.stride(1),
        k=k.data_ptr(), v=v.data_ptr(), kv_stride_b=k.stride(0), kv_stride_h=k.stride(1),
        log_beta=None if log_beta is None else log_beta.data_ptr(),
        pos=None if pos is None else pos.data_ptr(),
        meta_stride_b=0 if meta is None else meta.stride(0), meta_stride_h=0 if meta is None else meta.stride(1),
        len=len.data_ptr(), t=None if t is None else t.data_ptr(),
        B=B, Hq=Hq, Hkv=Hkv, d=d, cap=cap, scale=float(scale),
        num_splits=int(num_splits), split_len=int(split_len),
        o_part=None if o_part is None else o_part.data_ptr(),
        lse_part=None if lse_part is None else lse_part.data_ptr(), counters=None,
        o=o.data_ptr(), o_dtype=odt, lse=None if lse is None else lse.data_ptr(),
        evict_cand=None if evict_cand is None else _cand_ptr(evict_cand, B * Hkv * int(num_splits)))
    return a


def kvb_decode_attn_noalloc(q, k, v, log_beta, pos, len, t, o, lse=None, *, scale: float = 0.0,
                            num_splits: int = 1, split_len: int = 0, stream=None) -> None:
    """kvb_decode_attn for callers that cannot provide scratch device memory.

    Same inputs and outputs as kvb_decode_attn, without o_part/lse_part: the split
    states live in the library's fixed device array (NOALLOC_SCRATCH_BYTES per GPU), so the
    call allocates nothing. A problem whose split states do not fit raises KvbError (invalid
    argument). Calls that overlap on the GPU share that array and race: keep them on one
    stream. The first call on a device looks up the array's address; make it before any
    stream capture.
    """
    B, Hq, Hkv, d, cap = _decode_shapes(q, k, v, log_beta, pos, len, t, o, lse, num_splits)
    _need(q, torch.bfloat16, "q"); _need(k, torch.bfloat16, "k"); _need(v, torch.bfloat16, "v")
    if q.stride(2) != 1 or k.stride(3) != 1 or k.stride(2) != d or v.stride() != k.stride():
        raise ValueError("q/k/v: innermost dim contiguous, slot stride d, k and v with equal strides")
    _need(len, torch.int32, "len"); _contig(len, "len")
    if log_beta is not None:
        _need(log_beta, torch.float32, "log_beta")
        _need(pos, torch.int32, "pos")
        if log_beta.stride() != pos.stride() or log_beta.stride(2) != 1:
            raise ValueError("log_beta and pos need equal strides with slot stride 1")
        _need(t, torch.int32, "t")
    if t is not None:
        _need(t, torch.int32, "t"); _contig(t, "t")
    if o.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("o must be float32 or bfloat16")
    _contig(o, "o")
    if lse is not None:
        _need(lse, torch.float32, "lse"); _contig(lse, "lse")
    a = _lib.AttnArgs(
        q=q.data_ptr(), q_stride_b=q.stride(0), q_stride_h=q.stride(1),
        k=k.data_ptr(), v=v.data_ptr(), kv_stride_b=k.stride(0), kv_stride_h=k.stride(1),
        log_beta=None if log_beta is None else log_beta.data_ptr(),
        pos=None if pos is None else pos.data_ptr(),
        meta_stride_b=0 if pos is None else pos.stride(0),
        meta_stride_h=0 if pos is None else pos.stride(1),
        len=len.data_ptr(), t=None if t is None else t.data_ptr(),
        B=B, Hq=Hq, Hkv=Hkv, d=d, cap=cap, scale=float(scale),
        num_splits=int(num_splits), split_len=int(split_len), o_part=None, lse_part=None, counters=None,
        o=o.data_ptr(), o_dtype=_lib.KVB_OUT_F32 if o.dtype == torch.float32 else _lib.KVB_OUT_BF16,
        lse=None if lse is None else lse.data_ptr())
    _check(_lib.lib().kvb_decode_attn_noalloc(ctypes.byref(a), _stream(stream)), "kvb_decode_attn_noalloc")


def kvb_merge_states(o_in, lse_in, o_out, lse_out=None, *, stream=None) -> None:
    """Merge n attention states per row: o_in [n, R, d] f32 (d contiguous; any n/R strides),
    lse_in [n, R] f32 -> o_out [R, d], lse_out [R]."""
    _need(o_in, torch.float32, "o_in"); _need(lse_in, torch.float32, "lse_in")
    _need(o_out, torch.float32, "o_out"); _contig(o_out, "o_out")
    n, R, d = o_in.shape
    if o_in.stride(2) != 1 or tuple(lse_in.shape) != (n, R):
        raise ValueError("o_in [n, R, d] with d contiguous, lse_in [n, R]")
    if lse_out is not None:
        _need(lse_out, torch.float32, "lse_out"); _contig(lse_out, "lse_out")
    _check(_lib.lib().kvb_merge_states(_ptr(o_in), _ptr(lse_in), o_in.stride(0), o_in.stride(1),
                                       lse_in.stride(0), lse_in.stride(1), n, R, d, _ptr(o_out), _ptr(lse_out),
                                       _stream(stream)), "kvb_merge_states")


def kvb_evict_insert(k, v, log_beta, pos, len, k_new, v_new, log_beta_new, t, M: int, victim=None, *,
                     cand=None, cand_n: int = 0, stream=None) -> None:
    """Budget enforcement + insertion (in place); see kvb_evict_insert in include/kvb.h.
    k_new/v_new may both be None (only log_beta and pos are written); cand/cand_n: the
    candidates of the immediately preceding kvb_decode_attn on this cache, or None."""
    if k.dim() != 4:
        raise ValueError("k must be [B, Hkv, cap, d]")
    B, Hkv, cap, d = k.shape
    for name, x, shp in (("v", v, (B, Hkv, cap, d)), ("log_beta", log_beta, (B, Hkv, cap)),
                         ("pos", pos, (B, Hkv, cap)), ("len", len, (B, Hkv)), ("k_new", k_new, (B, Hkv, d)),
                         ("v_new", v_new, (B, Hkv, d)), ("log_beta_new", log_beta_new, (B, Hkv)),
                         ("t", t, (B,)), ("victim", victim, (B, Hkv))):
        _shape(x, shp, name)
    for name, x in (("k", k), ("v", v)):
        _need(x, torch.bfloat16, name); _contig(x, name)
    _need(pos, torch.int32, "pos"); _contig(pos, "pos")
    _need(len, torch.int32, "len"); _contig(len, "len")
    _need(t, torch.int32, "t"); _contig(t, "t")
    if log_beta is not None:
        _need(log_beta, torch.float32, "log_beta"); _contig(log_beta, "log_beta")
        _need(log_beta_new, torch.float32, "log_beta_new"); _contig(log_beta_new, "log_beta_new")
    for name, x in (("k_new", k_new), ("v_new", v_new)):
        if x is not None:
            _need(x, torch.bfloat16, name); _contig(x, name)
    if victim is not None:
        _need(victim, torch.int32, "victim"); _contig(victim, "victim")
    cp = None if cand is None else ctypes.c_void_p(_cand_ptr(cand, B * Hkv * int(cand_n)))
    _check(_lib.lib().kvb_evict_insert(_ptr(k), _ptr(v), _ptr(log_beta), _ptr(pos), _ptr(len), _ptr(k_new),
                                       _ptr(v_new), _ptr(log_beta_new), _ptr(t), B, Hkv, d, cap, int(M),
                                       _ptr(victim), cp, int(cand_n) if cand is not None else 0,
                                       _stream(stream)), "kvb_evict_insert")


def kvb_compact_blocks(k, v, pos, log_beta, len, rm_start, rm_len, *, stream=None) -> None:
    """In-place removal of slots [rm_start[b], +rm_len[b]) from every kv head of sequence b."""
    if k.dim() != 4:
        raise ValueError("k must be [B, Hkv, cap, d]")
    B, Hkv, cap, d = k.shape
    for name, x, shp in (("v", v, (B, Hkv, cap, d)), ("pos", pos, (B, Hkv, cap)), ("log_beta", log_beta, (B, Hkv, cap)),
                         ("len", len, (B, Hkv)), ("rm_start", rm_start, (B,)), ("rm_len", rm_len, (B,))):
        _shape(x, shp, name)
    for name, x in (("k", k), ("v", v)):
        _need(x, torch.bfloat16, name); _contig(x, name)
    for name, x in (("pos", pos), ("len", len), ("rm_start", rm_start), ("rm_len", rm_len)):
        _need(x, torch.int32, name); _contig(x, name)
    if log_beta is not None:
        _need(log_beta, torch.float32, "log_beta"); _contig(log_beta, "log_beta")
    _check(_lib.lib().kvb_compact_blocks(_ptr(k), _ptr(v), _ptr(pos), _ptr(log_beta), _ptr(len), _ptr(rm_start),
                                         _ptr(rm_len), B, Hkv, d, cap, _stream(stream)), "kvb_compact_blocks")


def kvb_asm_workspace_bytes(N: int, H: int, K: int) -> int:
    return int(_lib.lib().kvb_asm_workspace_bytes(N, H, K))


def kvb_asm_lookup_merge(q, qbar, abar, log_zbar, o_self, lse_self, idx, o, lse, workspace, *,
                         stream=None) -> None:
    """Attention-state-memory lookup and merge; see kvb_asm_lookup_merge(_grouped) in include/kvb.h.
    workspace: a uint8 CUDA tensor of at least kvb_asm_workspace_bytes(N, H, K) bytes.
    o=None: only idx is computed (abar, log_zbar, o_self, lse_self, lse may be None).
    qbar [H_tables, K, d] with H_tables dividing H: head h reads table h // (H // H_tables)."""
    _need(q, torch.bfloat16, "q"); _need(qbar, torch.float32, "qbar")
    if o is not None:
        _need(abar, torch.bfloat16, "abar"); _need(log_zbar, torch.float32, "log_zbar")
        _need(o_self, torch.float32, "o_self"); _need(lse_self, torch.float32, "lse_self")
        _need(o, torch.float32, "o")
    elif idx is None:
        raise KvbError("kvb_asm_lookup_merge: o=None (assignment only) needs idx")
    for name, x in (("q", q), ("qbar", qbar), ("abar", abar), ("log_zbar", log_zbar), ("o_self", o_self),
                    ("lse_self", lse_self), ("o", o), ("workspace", workspace)):
        if x is not None:
            _contig(x, name)
    if idx is not None:
        _need(idx, torch.int32, "idx"); _contig(idx, "idx")
    if lse is not None:
        _need(lse, torch.float32, "lse"); _contig(lse, "lse")
    N, H, d = q.shape
    Ht, K = qbar.shape[0], qbar.shape[1]
    nbytes = workspace.numel() * workspace.element_size()
    _check(_lib.lib().kvb_asm_lookup_merge_grouped(_ptr(q), _ptr(qbar), _ptr(abar), _ptr(log_zbar), _ptr(o_self),
                                                   _ptr(lse_self), N, H, Ht, K, d, _ptr(idx), _ptr(o), _ptr(lse),
                                                   _ptr(workspace), nbytes, _stream(stream)),
           "kvb_asm_lookup_merge_grouped")


kvb_asm_lookup_merge_grouped = kvb_asm_lookup_merge   # the table count is qbar's first dimension


def kvb_asm_planes_bytes(H_tables: int, K: int) -> int:
    return int(_lib.lib().kvb_asm_planes_bytes(H_tables, K))


def kvb_asm_prepare(qbar, planes=None, *, stream=None):
    """Prepare a memory for kvb_asm_lookup_merge_planes: qbar [H_tables, K, d] f32 -> planes (a uint8
    CUDA tensor of kvb_asm_planes_bytes(H_tables, K) bytes; allocated when None). Returns planes."""
    _need(qbar, torch.float32, "qbar"); _contig(qbar, "qbar")
    Ht, K, d = qbar.shape
    nbytes = kvb_asm_planes_bytes(Ht, K)
    if planes is None:
        planes = torch.empty(nbytes, dtype=torch.uint8, device=qbar.device)
    _contig(planes, "planes")
    if planes.numel() * planes.element_size() < nbytes:
        raise ValueError("planes buffer too small")
    _check(_lib.lib().kvb_asm_prepare(_ptr(qbar), Ht, K, d, _ptr(planes), planes.numel() * planes.element_size(),
                                      _stream(stream)), "kvb_asm_prepare")
    return planes


def kvb_asm_lookup_merge_planes(q, planes, H_tables: int, K: int, abar, log_zbar, o_self, lse_self, idx, o, lse,
                                workspace, *, stream=None) -> None:
    """kvb_asm_lookup_merge over a memory prepared by kvb_asm_prepare (H_tables tables of K entries)."""
    _need(q, torch.bfloat16, "q"); _contig(q, "q"); _contig(planes, "planes")
    N, H, d = q.shape
    if o is not None:
        _need(abar, torch.bfloat16, "abar"); _need(log_zbar, torch.float32, "log_zbar")
        _need(o_self, torch.float32, "o_self"); _need(lse_self, torch.float32, "lse_self")
        _need(o, torch.float32, "o")
        for name, x, shp in (("abar", abar, (H_tables, K, d)), ("log_zbar", log_zbar, (H_tables, K)),
                             ("o_self", o_self, (N, H, d)), ("lse_self", lse_self, (N, H)), ("o", o, (N, H, d))):
            _shape(x, shp, name)
            _contig(x, name)
    elif idx is None:
        raise ValueError("o=None (assignment only) needs idx")
    _shape(idx, (N, H), "idx")
    _shape(lse, (N, H), "lse")
    if idx is not None:
        _need(idx, torch.int32, "idx"); _contig(idx, "idx")
    if lse is not None:
        _need(lse, torch.float32, "lse"); _contig(lse, "lse")
    _contig(workspace, "workspace")
    _check(_lib.lib().kvb_asm_lookup_merge_planes(
        _ptr(q), _ptr(planes), planes.numel() * planes.element_size(), _ptr(abar), _ptr(log_zbar), _ptr(o_self),
        _ptr(lse_self), N, H, int(H_tables), int(K), d, _ptr(idx), _ptr(o), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)), "kvb_asm_lookup_merge_planes")


def kvb_asm_aggregate_workspace_bytes(H: int, K: int) -> int:
    return int(_lib.lib().kvb_asm_aggregate_workspace_bytes(H, K))


def kvb_asm_aggregate(q, a, lse, idx, qbar, abar, log_zbar, count, workspace, *, z_mean: bool = False,
                      stream=None) -> None:
    """Attention-aware aggregation (offline memory build); see kvb_asm_aggregate(_grouped) in
    include/kvb.h. a, lse None: only qbar (and count) are computed. qbar [H_tables, K, d]: the
    rows of head h feed table h // (H // H_tables). workspace: a uint8 CUDA tensor of at least
    kvb_asm_aggregate_workspace_bytes(H_tables, K) bytes."""
    _need(q, torch.bfloat16, "q"); _need(idx, torch.int32, "idx"); _need(qbar, torch.float32, "qbar")
    if (a is None) != (lse is None):
        raise KvbError("kvb_asm_aggregate: a and lse go together")
    if a is not None:
        _need(a, torch.float32, "a"); _need(lse, torch.float32, "lse")
        _need(abar, torch.bfloat16, "abar"); _need(log_zbar, torch.float32, "log_zbar")
    if count is not None:
        _need(count, torch.int32, "count")
    for name, x in (("q", q), ("a", a), ("lse", lse), ("idx", idx), ("qbar", qbar), ("abar", abar),
                    ("log_zbar", log_zbar), ("count", count), ("workspace", workspace)):
        if x is not None:
            _contig(x, name)
    M, H, d = q.shape
    Ht, K = qbar.shape[0], qbar.shape[1]
    nbytes = workspace.numel() * workspace.element_size()
    _check(_lib.lib().kvb_asm_aggregate_grouped(_ptr(q), _ptr(a), _ptr(lse), _ptr(idx), M, H, Ht, K, d,
                                                int(bool(z_mean)), _ptr(qbar), _ptr(abar), _ptr(log_zbar),
                                                _ptr(count), _ptr(workspace), nbytes, _stream(stream)),
           "kvb_asm_aggregate_grouped")


kvb_asm_aggregate_grouped = kvb_asm_aggregate   # the table count is qbar's first dimension


def kvb_asm_entries_bf16(qbar, q, *, stream=None) -> None:
    """qbar [H, K, d] f32 -> q [K, H, d] bf16; see kvb_asm_entries_bf16 in include/kvb.h."""
    _need(qbar, torch.float32, "qbar"); _need(q, torch.bfloat16, "q")
    _contig(qbar, "qbar"); _contig(q, "q")
    H, K, d = qbar.shape
    _check(_lib.lib().kvb_asm_entries_bf16(_ptr(qbar), H, K, d, _ptr(q), _stream(stream)), "kvb_asm_entries_bf16")


def kvb_asm_index_workspace_bytes(H: int, C: int) -> int:
    return int(_lib.lib().kvb_asm_index_workspace_bytes(H, C))


def kvb_asm_index_csr(idx, offsets, members, workspace, *, stream=None) -> None:
    """Cluster lists from an assignment idx [K, H] into offsets [H, C + 1], members [H, K];
    see kvb_asm_index_csr in include/kvb.h."""
    for name, x in (("idx", idx), ("offsets", offsets), ("members", members)):
        _need(x, torch.int32, name); _contig(x, name)
    _contig(workspace, "workspace")
    K, H = idx.shape
    C = offsets.shape[1] - 1
    nbytes = workspace.numel() * workspace.element_size()
    _check(_lib.lib().kvb_asm_index_csr(_ptr(idx), K, H, C, _ptr(offsets), _ptr(members), _ptr(workspace), nbytes,
                                        _stream(stream)), "kvb_asm_index_csr")


def kvb_asm_hier_workspace_bytes(N: int, H: int, m: int) -> int:
    return int(_lib.lib().kvb_asm_hier_workspace_bytes(N, H, m))


def kvb_asm_hier_lookup_merge(q, qhat, offsets, members, qbar, abar, log_zbar, o_self, lse_self, idx, o, lse,
                              workspace, m: int, *, stream=None) -> None:
    """Two-level attention-state-memory lookup and merge; see kvb_asm_hier_lookup_merge in
    include/kvb.h. workspace: a uint8 CUDA tensor of at least kvb_asm_hier_workspace_bytes(N, H, m)
    bytes."""
    _need(q, torch.bfloat16, "q"); _need(qhat, torch.float32, "qhat"); _need(offsets, torch.int32, "offsets")
    _need(members, torch.int32, "members"); _need(qbar, torch.float32, "qbar"); _need(abar, torch.bfloat16, "abar")
    _need(log_zbar, torch.float32, "log_zbar"); _need(o_self, torch.float32, "o_self")
    _need(lse_self, torch.float32, "lse_self"); _need(o, torch.float32, "o")
    for name, x in (("q", q), ("qhat", qhat), ("offsets", offsets), ("members", members), ("qbar", qbar),
                    ("abar", abar), ("log_zbar", log_zbar), ("o_self", o_self), ("lse_self", lse_self), ("o", o),
                    ("workspace", workspace)):
        _contig(x, name)
    if idx is not None:
        _need(idx, torch.int32, "idx"); _contig(idx, "idx")
    if lse is not None:
        _need(lse, torch.float32, "lse"); _contig(lse, "lse")
    N, H, d = q.shape
    K = qbar.shape[1]
    C = qhat.shape[1]
    nbytes = workspace.numel() * workspace.element_size()
    _check(_lib.lib().kvb_asm_hier_lookup_merge(_ptr(q), _ptr(qhat), _ptr(offsets), _ptr(members), _ptr(qbar),
                                                _ptr(abar), _ptr(log_zbar), _ptr(o_self), _ptr(lse_self), N, H, K,
                                                C, int(m), d, _ptr(idx), _ptr(o), _ptr(lse), _ptr(workspace),
                                                nbytes, _stream(stream)), "kvb_asm_hier_lookup_merge")


# ----------------------------------------------------------------------------------------------
# paged cache (see "Paged cache" in include/kvb.h)
# ----------------------------------------------------------------------------------------------

class PagedPool:
    """The device tensors of a paged cache: k_pages, v_pages [P, PAGE_SLOTS, d] bf16, log_beta_pages
    (None: beta = 1) and pos_pages [P, PAGE_SLOTS], table [B, Hkv, max_pages] int32, len [B, Hkv],
    free_pages [P], free_count [1]. Freshly made, call kvb_paged_reset() before use."""

    def __init__(self, B, Hkv, d, max_pages, num_pages, with_beta=True, device="cuda"):
        S = _lib.PAGE_SLOTS
        self.B, self.Hkv, self.d, self.max_pages, self.num_pages = B, Hkv, d, max_pages, num_pages
        self.k_pages = torch.zeros(num_pages, S, d, dtype=torch.bfloat16, device=device)
        self.v_pages = torch.zeros_like(self.k_pages)
        self.log_beta_pages = torch.zeros(num_pages, S, dtype=torch.float32, device=device) if with_beta else None
        self.pos_pages = torch.zeros(num_pages, S, dtype=torch.int32, device=device)
        self.table = torch.full((B, Hkv, max_pages), -1, dtype=torch.int32, device=device)
        self.len = torch.zeros(B, Hkv, dtype=torch.int32, device=device)
        self.free_pages = torch.zeros(num_pages, dtype=torch.int32, device=device)
        self.free_count = torch.zeros(1, dtype=torch.int32, device=device)

    def args(self, use_beta=True) -> "_lib.PagedCacheArgs":
        lb = self.log_beta_pages if use_beta else None
        return _lib.PagedCacheArgs(
            k_pages=self.k_pages.data_ptr(), v_pages=self.v_pages.data_ptr(),
            log_beta_pages=None if lb is None else lb.data_ptr(), pos_pages=self.pos_pages.data_ptr(),
            table=self.table.data_ptr(), len=self.len.data_ptr(), free_pages=self.free_pages.data_ptr(),
            free_count=self.free_count.data_ptr(), B=self.B, Hkv=self.Hkv, d=self.d, max_pages=self.max_pages,
            num_pages=self.num_pages)


def _pool(pool, use_beta=True):
    if not isinstance(pool, PagedPool):
        raise TypeError("pool must be a PagedPool")
    return ctypes.byref(pool.args(use_beta))


def kvb_paged_reset(pool, *, stream=None) -> None:
    """Every page free, every table entry -1, len 0."""
    _check(_lib.lib().kvb_paged_reset(_pool(pool), _stream(stream)), "kvb_paged_reset")


def kvb_paged_evict_insert(pool, k_new, v_new, log_beta_new, t, M: int, victim=None, *, cand=None, cand_n: int = 0,
                           stream=None) -> None:
    """Budget enforcement + insertion on a paged cache (kvb_evict_insert on the logical cache)."""
    B, Hkv, d = pool.B, pool.Hkv, pool.d
    for name, x, shp in (("k_new", k_new, (B, Hkv, d)), ("v_new", v_new, (B, Hkv, d)),
                         ("log_beta_new", log_beta_new, (B, Hkv)), ("t", t, (B,)), ("victim", victim, (B, Hkv))):
        _shape(x, shp, name)
    for name, x in (("k_new", k_new), ("v_new", v_new)):
        if x is not None:
            _need(x, torch.bfloat16, name); _contig(x, name)
    _need(t, torch.int32, "t"); _contig(t, "t")
    if pool.log_beta_pages is not None:
        _need(log_beta_new, torch.float32, "log_beta_new"); _contig(log_beta_new, "log_beta_new")
    if victim is not None:
        _need(victim, torch.int32, "victim"); _contig(victim, "victim")
    cp = None if cand is None else ctypes.c_void_p(_cand_ptr(cand, B * Hkv * int(cand_n)))
    _check(_lib.lib().kvb_paged_evict_insert(_pool(pool), _ptr(k_new), _ptr(v_new),
                                             _ptr(log_beta_new) if pool.log_beta_pages is not None else None,
                                             _ptr(t), int(M), _ptr(victim), cp, int(cand_n) if cand is not None else 0,
                                             _stream(stream)), "kvb_paged_evict_insert")


def kvb_paged_decode_attn(pool, q, t, o, lse=None, *, use_beta=True, scale: float = 0.0, num_splits: int = 1,
                          split_len: int = 0, o_part=None, lse_part=None, evict_cand=None, stream=None) -> None:
    """Decode attention over a paged cache (kvb_decode_attn on the logical cache). q [B, Hq, d] bf16
    contiguous; one split, or split_len a multiple of PAGE_SLOTS; the rest as kvb_decode_attn."""
    if q.dim() != 3:
        raise ValueError("q must be [B, Hq, d]")
    B, Hq, d = q.shape
    if B != pool.B or d != pool.d:
        raise ValueError("q must be [B, Hq, d] of the pool's B and d")
    for name, x, shp in (("t", t, (B,)), ("o", o, (B, Hq, d)), ("lse", lse, (B, Hq)),
                         ("o_part", o_part, (B, Hq, num_splits, d)), ("lse_part", lse_part, (B, Hq, num_splits))):
        _shape(x, shp, name)
    if num_splits > 1 and (o_part is None or lse_part is None):
        raise ValueError("num_splits > 1 needs o_part and lse_part (decode_workspace())")
    _need(q, torch.bfloat16, "q"); _contig(q, "q")
    if t is not None:
        _need(t, torch.int32, "t"); _contig(t, "t")
    if o.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("o must be float32 or bfloat16")
    _contig(o, "o")
    for name, x in (("lse", lse), ("o_part", o_part), ("lse_part", lse_part)):
        if x is not None:
            _need(x, torch.float32, name); _contig(x, name)
    cand = None if evict_cand is None else ctypes.c_void_p(_cand_ptr(evict_cand, B * pool.Hkv * int(num_splits)))
    _check(_lib.lib().kvb_paged_decode_attn(_pool(pool, use_beta), _ptr(q), _ptr(t), Hq, float(scale),
                                            int(num_splits), int(split_len), _ptr(o_part), _ptr(lse_part), _ptr(o),
                                            _lib.KVB_OUT_F32 if o.dtype == torch.float32 else _lib.KVB_OUT_BF16,
                                            _ptr(lse), cand, _stream(stream)), "kvb_paged_decode_attn")


def kvb_paged_compact_blocks(pool, rm_start, rm_len, *, stream=None) -> None:
    """In-place removal of slots [rm_start[b], +rm_len[b]) from every kv head of sequence b of a paged
    cache; pages past the new lengths return to the free stack."""
    for name, x in (("rm_start", rm_start), ("rm_len", rm_len)):
        _shape(x, (pool.B,), name)
        _need(x, torch.int32, name); _contig(x, name)
    _check(_lib.lib().kvb_paged_compact_blocks(_pool(pool), _ptr(rm_start), _ptr(rm_len), _stream(stream)),
           "kvb_paged_compact_blocks")
