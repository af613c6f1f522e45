"""Device-resident memory-bounded KV cache of one attention layer, and its decode step.

A decode step for the token at position t (per sequence) follows "Cache What
Lasts" section 2.1 at inference time: if the cache already holds M tokens the
token with the lowest beta_i^(t-i) is evicted and the new token takes its
slot (kvb_evict_insert); then the token attends over the <= M cached tokens,
itself included, with the retention-gated logits (kvb_decode_attn, split-K;
with several splits the same call launches the merge of the split states).
The attention also leaves, per split, the slot that the next position's
eviction would pick, so that the next insert reads candidates instead of
rescanning the cache.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (kvb_compact_blocks, kvb_decode_attn, kvb_decode_step, kvb_evict_insert, decode_workspace,
               evict_candidates)


def _dev(a, device):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


class BoundedKVCache:
    """K, V [B, Hkv, cap, d] bf16, log_beta [B, Hkv, cap] f32 (None: beta = 1), pos [B, Hkv, cap]
    int32, len [B, Hkv] int32, plus the split-K workspace for `num_splits` splits."""

    def __init__(self, B, Hq, Hkv, d, cap, M, num_splits=1, split_len=0, with_beta=True, device="cuda"):
        self.B, self.Hq, self.Hkv, self.d, self.cap, self.M = B, Hq, Hkv, d, cap, M
        self.num_splits, self.split_len = num_splits, split_len
        self.device = device
        self.k = torch.zeros(B, Hkv, cap, d, dtype=torch.bfloat16, device=device)
        self.v = torch.zeros_like(self.k)
        self.log_beta = torch.zeros(B, Hkv, cap, dtype=torch.float32, device=device) if with_beta else None
        self.pos = torch.zeros(B, Hkv, cap, dtype=torch.int32, device=device)
        self.len = torch.zeros(B, Hkv, dtype=torch.int32, device=device)
        self.victim = torch.zeros(B, Hkv, dtype=torch.int32, device=device)
        self.o_part = self.lse_part = None
        if num_splits > 1:
            self.o_part, self.lse_part = decode_workspace(B, Hq, d, num_splits, device)
        # eviction candidates for the next position, left by each attention pass; a fused step
        # reads one buffer and writes the other
        self.cand = evict_candidates(B, Hkv, num_splits, device)
        self.cand_next = evict_candidates(B, Hkv, num_splits, device)
        self.cand_valid = False
        # the caller's statement that every row holds M slots (set by from_host when the lengths
        # say so): then a step whose records are valid runs as one launch (kvb_decode_step)
        self.full = False

    @classmethod
    def from_host(cls, k, v, log_beta, pos, len_, Hq, M, num_splits=1, split_len=0, device="cuda"):
        B, Hkv, cap, d = k.shape
        c = cls(B, Hq, Hkv, d, cap, M, num_splits, split_len, log_beta is not None, device)
        c.k.copy_(_dev(k, device))
        c.v.copy_(_dev(v, device))
        if log_beta is not None:
            c.log_beta.copy_(_dev(log_beta, device))
        c.pos.copy_(_dev(pos, device))
        c.len.copy_(_dev(len_, device))
        c.full = bool(np.all(np.asarray(len_) == M))
        return c

    def insert(self, k_new, v_new, log_beta_new, t, stream=None):
        """Budget enforcement + insertion at position t. Uses the candidates of the attention at
        t - 1 when the last operation on the cache was that attention (the decode-step order)."""
        kvb_evict_insert(self.k, self.v, self.log_beta, self.pos, self.len, k_new, v_new,
                         log_beta_new if self.log_beta is not None else None, t, self.M, self.victim,
                         cand=self.cand if self.cand_valid else None, cand_n=self.num_splits, stream=stream)
        self.cand_valid = False

    def attend(self, q, t, o, lse=None, stream=None, use_beta=True):
        lb = self.log_beta if use_beta else None
        # candidates use the cache's own eviction score: only an attention with the same scoring
        # (bias on a retention cache, plain on a plain cache) can leave them
        same_scoring = (lb is not None) == (self.log_beta is not None)
        cand = self.cand if (same_scoring and t is not None) else None
        kvb_decode_attn(q, self.k, self.v, lb, self.pos, self.len, t if (lb is not None or t is not None) else None,
                        o, lse, num_splits=self.num_splits, split_len=self.split_len, o_part=self.o_part,
                        lse_part=self.lse_part, evict_cand=cand, stream=stream)
        # the records describe this attention's cache state only: an attention that leaves none
        # makes earlier records stale for the next insertion
        self.cand_valid = cand is not None

    def step(self, q, k_new, v_new, log_beta_new, t, o, lse=None, stream=None):
        """One decode step: budget enforcement + insertion, then attention. One launch
        (kvb_decode_step) when the cache is full and the last attention left the records for
        this position; else two (kvb_evict_insert, kvb_decode_attn)."""
        if self.full and self.cand_valid and t is not None:
            kvb_decode_step(q, self.k, self.v, self.log_beta, self.pos, self.len, t, o, lse, k_new, v_new,
                            log_beta_new if self.log_beta is not None else None, self.M, self.cand,
                            self.cand_next, victim=self.victim, num_splits=self.num_splits,
                            split_len=self.split_len, o_part=self.o_part, lse_part=self.lse_part, stream=stream)
            self.cand, self.cand_next = self.cand_next, self.cand
            return
        self.insert(k_new, v_new, log_beta_new, t, stream)
        self.attend(q, t, o, lse, stream)

    def compact(self, rm_start, rm_len, stream=None):
        kvb_compact_blocks(self.k, self.v, self.pos, self.log_beta, self.len, rm_start, rm_len, stream=stream)
        self.cand_valid = False
        self.full = False

    def kv_bytes_read(self) -> int:
        """Bytes of K, V (and log_beta, pos when the bias is on) that one attention pass reads."""
        n = int(self.len.sum().item())
        per_slot = 2 * self.d * 2 + (8 if self.log_beta is not None else 0)
        return n * per_slot


class PagedKVCache:
    """The cache of BoundedKVCache kept in pages of PAGE_SLOTS slots from one pool (kvb_paged_*):
    the same decode step on the same logical cache, with memory for the pages in use instead of
    `cap` slots per (sequence, kv head). Splits start on pages: num_splits == 1 or split_len a
    multiple of PAGE_SLOTS."""

    def __init__(self, B, Hq, Hkv, d, max_pages, num_pages, M, num_splits=1, split_len=0, with_beta=True,
                 device="cuda"):
        from . import PagedPool, kvb_paged_reset
        self.B, self.Hq, self.Hkv, self.d, self.M = B, Hq, Hkv, d, M
        self.num_splits, self.split_len = num_splits, split_len
        self.pool = PagedPool(B, Hkv, d, max_pages, num_pages, with_beta, device)
        kvb_paged_reset(self.pool)
        self.victim = torch.zeros(B, Hkv, dtype=torch.int32, device=device)
        self.o_part = self.lse_part = None
        if num_splits > 1:
            self.o_part, self.lse_part = decode_workspace(B, Hq, d, num_splits, device)
        self.cand = evict_candidates(B, Hkv, num_splits, device)
        self.cand_valid = False

    @property
    def len(self):
        return self.pool.len

    def reset(self):
        from . import kvb_paged_reset
        kvb_paged_reset(self.pool)
        self.cand_valid = False

    def insert(self, k_new, v_new, log_beta_new, t, stream=None):
        from . import kvb_paged_evict_insert
        kvb_paged_evict_insert(self.pool, k_new, v_new, log_beta_new, t, self.M, self.victim,
                               cand=self.cand if self.cand_valid else None, cand_n=self.num_splits, stream=stream)
        self.cand_valid = False

    def attend(self, q, t, o, lse=None, stream=None, use_beta=True):
        from . import kvb_paged_decode_attn
        with_beta = self.pool.log_beta_pages is not None
        same_scoring = use_beta or not with_beta
        cand = self.cand if (same_scoring and t is not None) else None
        kvb_paged_decode_attn(self.pool, q, t, o, lse, use_beta=use_beta, num_splits=self.num_splits,
                              split_len=self.split_len, o_part=self.o_part, lse_part=self.lse_part,
                              evict_cand=cand, stream=stream)
        self.cand_valid = cand is not None

    def step(self, q, k_new, v_new, log_beta_new, t, o, lse=None, stream=None):
        self.insert(k_new, v_new, log_beta_new, t, stream)
        self.attend(q, t, o, lse, stream)

    def compact(self, rm_start, rm_len, stream=None):
        from . import kvb_paged_compact_blocks
        kvb_paged_compact_blocks(self.pool, rm_start, rm_len, stream=stream)
        self.cand_valid = False

    def pages_in_use(self) -> int:
        return self.pool.num_pages - int(self.pool.free_count.item())
