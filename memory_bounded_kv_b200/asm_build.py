"""Offline build of an attention-state memory on the GPU ("Context Memorization", core method
steps 1-2), from calibration queries and their attention states over the prefix.

  q   [M, H, d] bf16  calibration queries (per head)
  a   [M, H, d] f32   their attention outputs over the prefix (e.g. kvb_decode_attn's o)
  lse [M, H]    f32   ln Z of those attentions (kvb_decode_attn's lse)

Clustering: Lloyd's iteration under the cosine, the lookup's own similarity. The assignment step
is kvb_asm_lookup_merge without a merge (o=None: the cosine argmax over the current centroids,
on the tensor cores), the update step is kvb_asm_aggregate without states (the mean of every
cluster's queries). The centroids start as the queries init_rows[h] of each head. Then the states
are aggregated over the final clusters (mean of the queries, merge-fold of (a, Z)). Every step is
a kernel of this library; this module only allocates and sequences the calls.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (kvb_asm_aggregate, kvb_asm_aggregate_workspace_bytes, kvb_asm_entries_bf16, kvb_asm_index_csr,
               kvb_asm_index_workspace_bytes, kvb_asm_lookup_merge, kvb_asm_workspace_bytes)


def _initial_assignment(init_rows, M: int, device) -> torch.Tensor:
    """idx [M, H] with query init_rows[h, k] in cluster k and every other query in none."""
    init_rows = np.asarray(init_rows)
    H, K = init_rows.shape
    idx = np.full((M, H), -1, np.int32)
    for h in range(H):
        if len(set(init_rows[h].tolist())) != K or init_rows[h].min() < 0 or init_rows[h].max() >= M:
            raise ValueError("init_rows[h] must hold K distinct query rows")
        idx[init_rows[h], h] = np.arange(K, dtype=np.int32)
    return torch.from_numpy(idx).to(device)


def asm_kmeans(q: torch.Tensor, init_rows, iters: int, stream=None):
    """Lloyd under the cosine. Returns (idx [M, H] int32, centroids [H, K, d] f32) after the
    assignment to the centroids of `iters` updates (the sequence: start, assign, then `iters`
    times update and assign)."""
    M, H, d = q.shape
    K = np.asarray(init_rows).shape[1]
    dev = q.device
    cent = torch.empty(H, K, d, dtype=torch.float32, device=dev)
    ws_agg = torch.empty(kvb_asm_aggregate_workspace_bytes(H, K), dtype=torch.uint8, device=dev)
    ws_lk = torch.empty(kvb_asm_workspace_bytes(M, H, K), dtype=torch.uint8, device=dev)
    idx = torch.empty(M, H, dtype=torch.int32, device=dev)
    # the starting centroids are the chosen queries: the mean of one-member clusters
    kvb_asm_aggregate(q, None, None, _initial_assignment(init_rows, M, dev), cent, None, None, None, ws_agg,
                      stream=stream)
    kvb_asm_lookup_merge(q, cent, None, None, None, None, idx, None, None, ws_lk, stream=stream)
    for _ in range(iters):
        kvb_asm_aggregate(q, None, None, idx, cent, None, None, None, ws_agg, stream=stream)
        kvb_asm_lookup_merge(q, cent, None, None, None, None, idx, None, None, ws_lk, stream=stream)
    return idx, cent


def asm_build(q: torch.Tensor, a: torch.Tensor, lse: torch.Tensor, init_rows, iters: int,
              z_mean: bool = False, stream=None):
    """Clusters the calibration queries (asm_kmeans) and aggregates their states.
    Returns (qbar [H, K, d] f32, abar [H, K, d] bf16, log_zbar [H, K] f32, count [H, K] int32,
    idx [M, H] int32): the memory that kvb_asm_lookup_merge reads, and the final clusters."""
    M, H, d = q.shape
    K = np.asarray(init_rows).shape[1]
    dev = q.device
    idx, _ = asm_kmeans(q, init_rows, iters, stream)
    qbar = torch.empty(H, K, d, dtype=torch.float32, device=dev)
    abar = torch.empty(H, K, d, dtype=torch.bfloat16, device=dev)
    log_zbar = torch.empty(H, K, dtype=torch.float32, device=dev)
    count = torch.empty(H, K, dtype=torch.int32, device=dev)
    ws = torch.empty(kvb_asm_aggregate_workspace_bytes(H, K), dtype=torch.uint8, device=dev)
    kvb_asm_aggregate(q, a, lse, idx, qbar, abar, log_zbar, count, ws, z_mean=z_mean, stream=stream)
    return qbar, abar, log_zbar, count, idx


def asm_index(qbar: torch.Tensor, init_rows, iters: int, stream=None):
    """Two-level index of a memory for kvb_asm_hier_lookup_merge: the entries qbar [H, K, d] f32,
    as bf16 queries (kvb_asm_entries_bf16), are clustered into C = init_rows.shape[1] groups per
    head (asm_kmeans, starting from the entries init_rows[h]); the groups' means are the
    first-level centroids and kvb_asm_index_csr lists each group's entries in increasing order.
    Returns (qhat [H, C, d] f32, offsets [H, C + 1] int32, members [H, K] int32, idx [K, H] int32)."""
    H, K, d = qbar.shape
    C = np.asarray(init_rows).shape[1]
    dev = qbar.device
    q = torch.empty(K, H, d, dtype=torch.bfloat16, device=dev)
    kvb_asm_entries_bf16(qbar, q, stream=stream)
    idx, qhat = asm_kmeans(q, init_rows, iters, stream)
    offsets = torch.empty(H, C + 1, dtype=torch.int32, device=dev)
    members = torch.empty(H, K, dtype=torch.int32, device=dev)
    ws = torch.empty(kvb_asm_index_workspace_bytes(H, C), dtype=torch.uint8, device=dev)
    kvb_asm_index_csr(idx, offsets, members, ws, stream=stream)
    return qhat, offsets, members, idx
