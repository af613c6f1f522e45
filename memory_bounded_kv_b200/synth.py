"""Seeded synthetic inputs for the memory-bounded KV decode path.

This module holds random draws, their rounding to the storage types, and the
schedules (positions, lengths, block boundaries) that the five workloads
prescribe. It holds none of the method's arithmetic: no attention, no merge,
no eviction score, no lookup. Both the CUDA path (through the tests and the
bench) and the CPU oracle take their inputs from here, so that both sides see
identical bits.

Every draw comes from ``numpy.random.default_rng([seed, stream, ...])`` so a
single step's inputs can be regenerated without replaying earlier steps.

Workloads (sizes and distributions as the retention-gated, memento and
attention-state-memory pages describe them; see each function):

1. tiny retention-gated decode          ``decode_workload(1)``
2. Qwen3-8B-shaped layer decode step    ``decode_workload(2)``
3. long-context bounded cache           ``decode_workload(3)`` + ``stream_log_beta``
4. attention-state-memory lookup        ``asm_workload()``
5. memento-style block compaction       ``memento_workload()``
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# stream ids inside one seed
_S_CACHE, _S_STEP, _S_STREAM, _S_SCHED = 0, 1, 2, 10


def rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), *[int(s) for s in stream]])


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the bits as uint16."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(g: np.random.Generator, shape) -> np.ndarray:
    """N(0, 1) draws stored as bf16 bits."""
    return to_bf16_bits(g.standard_normal(shape, dtype=np.float32))


def log_beta(g: np.random.Generator, shape, mu: float = 2.0, sigma: float = 1.5) -> np.ndarray:
    """log of a retention score beta = sigmoid(x), x ~ N(mu, sigma), as float32.

    The retention gate that would produce beta is a trained network and is not
    part of this library; the workloads draw beta from sigmoid(N(2, 1.5)). The
    log is taken once here, in double (log sigmoid(x) = -log(1 + e^-x)), and
    rounded to float32, which is the type the library takes.
    """
    x = g.normal(mu, sigma, size=shape)
    return (-np.logaddexp(0.0, -x)).astype(np.float32)


# --------------------------------------------------------------------------
# decode workloads: tiny (1), Qwen3-8B-shaped layer (2), long context (3)
# --------------------------------------------------------------------------

@dataclass
class DecodeWorkload:
    """A bounded-cache decode workload: a prefilled cache and per-step token inputs.

    Cache layout: k, v [B, Hkv, cap, d] bf16 bits; log_beta, pos [B, Hkv, cap];
    len [B, Hkv]. Slots at or beyond len hold zeros.
    """
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    d: int
    M: int
    cap: int
    t0: int                 # position of the first decoded token
    steps: int              # decode steps the workload prescribes
    splits: tuple = (1,)
    k: np.ndarray = field(repr=False, default=None)
    v: np.ndarray = field(repr=False, default=None)
    log_beta: np.ndarray = field(repr=False, default=None)
    pos: np.ndarray = field(repr=False, default=None)
    len: np.ndarray = field(repr=False, default=None)

    def step_inputs(self, step: int) -> dict:
        """Token inputs of decode step `step` (position t0 + step)."""
        g = rng(self.seed, _S_STEP, step)
        q = normal_bf16(g, (self.B, self.Hq, self.d))
        k_new = normal_bf16(g, (self.B, self.Hkv, self.d))
        v_new = normal_bf16(g, (self.B, self.Hkv, self.d))
        lb_new = log_beta(g, (self.B, self.Hkv))
        t = np.full((self.B,), self.t0 + step, dtype=np.int32)
        return dict(q=q, k_new=k_new, v_new=v_new, log_beta_new=lb_new, t=t)


_DECODE_CONFIGS = {
    # tiny retention-gated decode: prefill 256 then 512 steps with evict-on-overflow
    1: dict(name="tiny-retention-decode B1 Hq8 Hkv2 d64 M256", seed=0, B=1, Hq=8, Hkv=2, d=64,
            M=256, cap=256, prefill=256, steps=512, splits=(1, 4)),
    # Qwen3-8B-shaped layer: full budget 4096, 1024 steps of evict+insert+attend
    2: dict(name="qwen3-8b-layer B32 Hq32 Hkv8 d128 M4096", seed=2, B=32, Hq=32, Hkv=8, d=128,
            M=4096, cap=4096, prefill=4096, steps=1024, splits=(1,)),
    # long context 131072 held in 8192 slots, 64 splits
    3: dict(name="long-context B4 Hq32 Hkv8 d128 M8192 ctx131072", seed=3, B=4, Hq=32, Hkv=8, d=128,
            M=8192, cap=8192, prefill=8192, steps=64, splits=(64,)),
}

CONFIG3_LOGICAL_T = 131072


def decode_workload(cfg: int, B: int | None = None, prefill: int | None = None,
                    seed: int | None = None) -> DecodeWorkload:
    """Prefilled cache of decode workload 1 (tiny), 2 (Qwen3-8B-shaped) or 3 (long context).

    Prefill writes positions 0..prefill-1 into slots 0..prefill-1 (no eviction
    while the cache is within budget). `B` may shrink the batch (the first B
    sequences of the full draw are not reproduced; a smaller B is a different,
    smaller workload of the same shape). `seed` replaces the workload's own seed.

    For the long-context workload the returned cache is the starting point of the streaming
    build (positions 0..8191); the caller streams positions 8192..131071
    through budget enforcement with ``stream_log_beta`` (30 blocks of 4096
    positions) and then redraws the surviving slots' K/V with ``long_context_kv``.
    """
    c = dict(_DECODE_CONFIGS[cfg])
    if B is not None:
        c["B"] = B
    if seed is not None:
        c["seed"] = int(seed)
    P = c.pop("prefill")
    if prefill is not None:
        P = prefill
    w = DecodeWorkload(t0=P, **c)
    g = rng(w.seed, _S_CACHE)
    shape = (w.B, w.Hkv, w.cap)
    w.k = np.zeros(shape + (w.d,), np.uint16)
    w.v = np.zeros(shape + (w.d,), np.uint16)
    w.k[:, :, :P] = normal_bf16(g, (w.B, w.Hkv, P, w.d))
    w.v[:, :, :P] = normal_bf16(g, (w.B, w.Hkv, P, w.d))
    w.log_beta = np.zeros(shape, np.float32)
    w.log_beta[:, :, :P] = log_beta(g, (w.B, w.Hkv, P))
    w.pos = np.zeros(shape, np.int32)
    w.pos[:, :, :P] = np.arange(P, dtype=np.int32)
    w.len = np.full((w.B, w.Hkv), P, np.int32)
    if cfg == 3:
        w.t0 = CONFIG3_LOGICAL_T
    return w


STREAM_BLOCK = 4096


def stream_log_beta(w: DecodeWorkload, block: int) -> np.ndarray:
    """log beta of the config-3 streaming build, positions [cap + block*4096, +4096), as [4096, B, Hkv]."""
    g = rng(w.seed, _S_STREAM, block)
    return log_beta(g, (STREAM_BLOCK, w.B, w.Hkv))


def long_context_kv(w: DecodeWorkload) -> tuple[np.ndarray, np.ndarray]:
    """K/V of the slots that survive the config-3 streaming build (drawn after the build)."""
    g = rng(w.seed, _S_CACHE, 1)
    shape = (w.B, w.Hkv, w.cap, w.d)
    return normal_bf16(g, shape), normal_bf16(g, shape)


# --------------------------------------------------------------------------
# attention-state memory lookup workload
# --------------------------------------------------------------------------

@dataclass
class ASMWorkload:
    """Per-head memory of K centroids plus N query tokens with their own causal self-attention.

    qbar [H, K, d] float32 (unit rows), abar [H, K, d] bf16 bits, log_zbar [H, K] float32,
    q [N, H, d] bf16 bits; self cache k, v [1, Hkv, L, d] shared by all N queries (batch
    stride 0); query j sits at position L - N + j and sees keys 0 .. L - N + j (len = L - N + j + 1).
    """
    seed: int
    N: int
    H: int
    Hkv: int
    K: int
    d: int
    L: int
    qbar: np.ndarray = field(repr=False, default=None)
    abar: np.ndarray = field(repr=False, default=None)
    log_zbar: np.ndarray = field(repr=False, default=None)
    q: np.ndarray = field(repr=False, default=None)
    k: np.ndarray = field(repr=False, default=None)
    v: np.ndarray = field(repr=False, default=None)
    pos: np.ndarray = field(repr=False, default=None)
    len: np.ndarray = field(repr=False, default=None)
    t: np.ndarray = field(repr=False, default=None)


def asm_workload(N: int = 256, H: int = 32, Hkv: int = 8, K: int = 4096, d: int = 128,
                 L: int = 2048, seed: int = 4) -> ASMWorkload:
    w = ASMWorkload(seed=seed, N=N, H=H, Hkv=Hkv, K=K, d=d, L=L)
    g = rng(seed, _S_CACHE)
    x = g.standard_normal((H, K, d))
    w.qbar = (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)
    w.abar = normal_bf16(g, (H, K, d))
    w.log_zbar = g.uniform(5.0, 12.0, (H, K)).astype(np.float32)
    w.q = normal_bf16(g, (N, H, d))
    w.k = normal_bf16(g, (1, Hkv, L, d))
    w.v = normal_bf16(g, (1, Hkv, L, d))
    w.pos = np.arange(L, dtype=np.int32).reshape(1, 1, L).repeat(Hkv, axis=1)
    first = L - N
    w.t = (first + np.arange(N)).astype(np.int32)
    w.len = np.repeat((w.t + 1)[:, None], Hkv, axis=1).astype(np.int32)
    return w


@dataclass
class ASMIndex:
    """A clustered attention-state memory with its two-level index.

    Per head: C cluster directions u_c (unit, float32) serve as the first-level centroids
    qhat [H, C, d]; cluster c holds a ragged number of entries (sizes around K / C, every entry
    in exactly one cluster, ids scattered over [0, K)), each entry qbar_k = unit(u_c + sigma g).
    members [H, K] int32 lists the entries cluster by cluster, offsets [H, C + 1] int32 bounds
    each cluster's run. Queries are unit(u_c' + sigma_q g) for a random cluster c', in bf16.
    """
    seed: int
    N: int
    H: int
    K: int
    C: int
    d: int
    qhat: np.ndarray = field(repr=False, default=None)
    offsets: np.ndarray = field(repr=False, default=None)
    members: np.ndarray = field(repr=False, default=None)
    qbar: np.ndarray = field(repr=False, default=None)
    abar: np.ndarray = field(repr=False, default=None)
    log_zbar: np.ndarray = field(repr=False, default=None)
    q: np.ndarray = field(repr=False, default=None)
    o_self: np.ndarray = field(repr=False, default=None)
    lse_self: np.ndarray = field(repr=False, default=None)


def _unit(x: np.ndarray) -> np.ndarray:
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    return x / np.where(n > 0, n, 1.0)


def asm_index_workload(N: int = 1, H: int = 32, K: int = 4096, C: int = 64, d: int = 128,
                       sigma: float = 2.5, sigma_q: float = 2.0, seed: int = 6) -> ASMIndex:
    w = ASMIndex(seed=seed, N=N, H=H, K=K, C=C, d=d)
    g = rng(seed, _S_CACHE)
    u = _unit(g.standard_normal((H, C, d)))
    w.qhat = u.astype(np.float32)
    w.qbar = np.zeros((H, K, d), np.float32)
    w.members = np.zeros((H, K), np.int32)
    w.offsets = np.zeros((H, C + 1), np.int32)
    for h in range(H):
        # ragged sizes: a multinomial split of K over the C clusters
        sizes = g.multinomial(K, np.full(C, 1.0 / C))
        w.offsets[h, 1:] = np.cumsum(sizes)
        ids = g.permutation(K).astype(np.int32)
        w.members[h] = ids
        owner = np.repeat(np.arange(C), sizes)          # cluster of the i-th listed entry
        x = u[h, owner] + sigma * g.standard_normal((K, d)) / np.sqrt(d)
        w.qbar[h, ids] = _unit(x).astype(np.float32)
    w.abar = normal_bf16(g, (H, K, d))
    w.log_zbar = g.uniform(5.0, 12.0, (H, K)).astype(np.float32)
    gq = rng(seed, _S_STEP)
    target = gq.integers(0, C, (N, H))
    xq = u[np.arange(H)[None, :], target] + sigma_q * gq.standard_normal((N, H, d)) / np.sqrt(d)
    w.q = to_bf16_bits(_unit(xq).astype(np.float32))
    w.o_self = gq.standard_normal((N, H, d)).astype(np.float32)
    w.lse_self = gq.uniform(3.0, 9.0, (N, H)).astype(np.float32)
    return w


# --------------------------------------------------------------------------
# memento-style block compaction (sawtooth cache)
# --------------------------------------------------------------------------

@dataclass
class MementoWorkload:
    """Per sequence: nblk x (thinking block ~ Geometric(1/mean_block), memento ~ U{lo..hi}).

    Token j of sequence b has position j. After decoding the last token of memento i
    (attention included), block i's slot range is removed from the cache in place:
    [sum(mem[b, :i]), + blk[b, i]). A finished sequence is inactive (t = -1).
    """
    seed: int
    B: int
    Hq: int
    Hkv: int
    d: int
    blk: np.ndarray = field(repr=False, default=None)     # [B, nblk] int
    mem: np.ndarray = field(repr=False, default=None)     # [B, nblk] int
    total: np.ndarray = field(repr=False, default=None)   # [B] tokens per sequence
    cap: int = 0
    pool: int = 64

    @property
    def steps(self) -> int:
        return int(self.total.max())

    def step_inputs(self, step: int) -> dict:
        """Token inputs of step `step`: q, k_new, v_new for every sequence, drawn from a pool of
        `pool` seeded draws (step s uses draw s mod pool); t = step for active sequences, -1 after."""
        g = rng(self.seed, _S_STEP, step % self.pool)
        q = normal_bf16(g, (self.B, self.Hq, self.d))
        k_new = normal_bf16(g, (self.B, self.Hkv, self.d))
        v_new = normal_bf16(g, (self.B, self.Hkv, self.d))
        t = np.where(step < self.total, step, -1).astype(np.int32)
        return dict(q=q, k_new=k_new, v_new=v_new, t=t)

    def compaction(self, step: int) -> tuple[np.ndarray, np.ndarray]:
        """(rm_start [B], rm_len [B]) to apply after the attention of `step` (zeros = no-op)."""
        ends = np.cumsum(self.blk + self.mem, axis=1) - 1          # last token of memento i
        start = np.zeros(self.B, np.int32)
        ln = np.zeros(self.B, np.int32)
        hit = ends == step
        for b, i in zip(*np.nonzero(hit)):
            start[b] = int(self.mem[b, :i].sum())
            ln[b] = int(self.blk[b, i])
        return start, ln

    def compaction_steps(self) -> np.ndarray:
        return np.unique(np.cumsum(self.blk + self.mem, axis=1) - 1)

    def len_trajectory(self) -> np.ndarray:
        """[steps, B] int64: every sequence's length after the insertion of each step (before that
        step's compaction); finished sequences keep their mementos."""
        steps = np.arange(self.steps)
        ends = np.cumsum(self.blk + self.mem, axis=1) - 1                  # [B, nblk] compaction steps
        out = np.zeros((self.steps, self.B), np.int64)
        for b in range(self.B):
            # blocks removed before step i: compactions at steps < i
            removed = np.zeros(self.steps + 1, np.int64)
            np.add.at(removed, ends[b] + 1, self.blk[b])
            removed = np.cumsum(removed)[: self.steps]
            out[:, b] = np.where(steps < self.total[b], steps + 1 - removed, self.mem[b].sum())
        return out

    def peak_pages(self, page: int = 64) -> int:
        """The most pages of `page` slots a paged cache of this schedule holds at once (all kv heads)."""
        n = self.len_trajectory()
        return int((self.Hkv * (-(-n // page))).sum(axis=1).max())

    def cache_len(self, step: int) -> np.ndarray:
        """len of every sequence after the insertion of step `step` and before its compaction."""
        out = np.zeros(self.B, np.int64)
        for b in range(self.B):
            if step >= self.total[b]:
                out[b] = self.mem[b].sum()
                continue
            bounds = np.cumsum(self.blk[b] + self.mem[b])
            i = int(np.searchsorted(bounds, step, side="right"))
            begin = 0 if i == 0 else int(bounds[i - 1])
            out[b] = int(self.mem[b, :i].sum()) + (step - begin + 1)
        return out


def memento_workload(B: int = 64, Hq: int = 32, Hkv: int = 8, d: int = 128, nblk: int = 9,
                     mean_block: float = 1500.0, mem_lo: int = 120, mem_hi: int = 180,
                     seed: int = 5) -> MementoWorkload:
    w = MementoWorkload(seed=seed, B=B, Hq=Hq, Hkv=Hkv, d=d)
    blk = np.zeros((B, nblk), np.int64)
    mem = np.zeros((B, nblk), np.int64)
    for b in range(B):
        g = rng(seed, _S_SCHED, b)
        blk[b] = g.geometric(1.0 / mean_block, nblk)
        mem[b] = g.integers(mem_lo, mem_hi + 1, nblk)
    w.blk, w.mem = blk, mem
    w.total = (blk + mem).sum(axis=1)
    # capacity = the largest concurrent length: earlier mementos + current block + its memento
    prev = np.concatenate([np.zeros((B, 1), np.int64), np.cumsum(mem, axis=1)[:, :-1]], axis=1)
    need = int((prev + blk + mem).max())
    w.cap = int(-(-need // 64) * 64)
    return w
