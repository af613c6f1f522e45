"""Oracle of the attention-state-memory offline build: attention-aware aggregation and the
Lloyd clustering of calibration queries ("Context Memorization", core method steps 1-2).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py). Plain numpy in float64; bf16 inputs are
uint16 bit patterns. Readings: the aggregated Z is the sum over the cluster (the merge operator
sums Z), with a switch for the mean; the clustering is Lloyd's iteration with the cosine as the
similarity (the lookup's own measure): assign every query to the centroid of largest cosine (the
lower index on ties), then move every centroid to the mean of its queries (an empty cluster gets
the zero vector, which no query with a positive cosine elsewhere picks again).
"""
from __future__ import annotations

import numpy as np


def _bf16(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def asm_aggregate(q, a, lse, idx, K: int, z_mean: bool = False):
    """Per head h and cluster k, over the members S = {i : idx[i, h] == k} (idx < 0: no cluster):
      qbar[h, k] = mean of q[i, h]                                   (core method step 2)
      (abar, Zbar)[h, k] = merge-fold of (a[i, h], Z[i, h]):  Zbar = sum Z_i,
                           abar = sum Z_i a_i / Zbar            (the page's merge operator)
      log_zbar = ln Zbar (minus ln |S| with z_mean); an empty cluster: 0, 0, -inf.
    q [M, H, d] bf16 bits; a [M, H, d]; lse [M, H] (ln Z); idx [M, H] int.
    a / lse may be None: then abar / log_zbar are None.
    Returns qbar [H, K, d], abar [H, K, d], log_zbar [H, K] (float64), count [H, K]."""
    qf = _bf16(q)
    M, H, d = qf.shape
    idx = np.asarray(idx)
    qbar = np.zeros((H, K, d))
    count = np.zeros((H, K), np.int64)
    abar = None if a is None else np.zeros((H, K, d))
    lz = None if lse is None else np.full((H, K), -np.inf)
    a64 = None if a is None else np.asarray(a, np.float64)
    l64 = None if lse is None else np.asarray(lse, np.float64)
    for h in range(H):
        for k in range(K):
            S = np.nonzero(idx[:, h] == k)[0]
            count[h, k] = len(S)
            if len(S) == 0:
                continue
            qbar[h, k] = qf[S, h].mean(axis=0)
            if a64 is None:
                continue
            m = l64[S, h].max()
            if m == -np.inf:          # every member's Z is 0: the merge identity
                continue
            w = np.exp(l64[S, h] - m)
            lz[h, k] = m + np.log(w.sum()) - (np.log(len(S)) if z_mean else 0.0)
            abar[h, k] = (w[:, None] * a64[S, h]).sum(axis=0) / w.sum()
    return qbar, abar, lz, count


def cosine_assign(q, cent):
    """idx[i, h] = argmax_k cos(q[i, h], cent[h, k]) (the first index among equal values;
    cos = 0 when either vector is zero). q [M, H, d] bf16 bits; cent [H, K, d]."""
    qf = _bf16(q)
    M, H, d = qf.shape
    c = np.asarray(cent, np.float64)
    idx = np.zeros((M, H), np.int32)
    for h in range(H):
        qn = np.linalg.norm(qf[:, h], axis=1)
        cn = np.linalg.norm(c[h], axis=1)
        dots = qf[:, h] @ c[h].T
        den = qn[:, None] * cn[None, :]
        cos = np.where(den > 0, dots / np.where(den > 0, den, 1.0), 0.0)
        idx[:, h] = np.argmax(cos, axis=1)
    return idx


def asm_kmeans(q, init_rows, iters: int):
    """Lloyd's iteration under the cosine, per head: centroids start as the queries init_rows[h]
    (K of them), then `iters` times assign (cosine_assign) and move the centroids to their
    clusters' means. Returns (idx [M, H] of the last assignment, centroids [H, K, d])."""
    qf = _bf16(q)
    M, H, d = qf.shape
    init_rows = np.asarray(init_rows)
    K = init_rows.shape[1]
    cent = np.stack([qf[init_rows[h], h] for h in range(H)])
    idx = cosine_assign(q, cent)
    for _ in range(iters):
        cent, _, _, _ = asm_aggregate(q, None, None, idx, K)
        idx = cosine_assign(q, cent)
    return idx, cent


def asm_index(qbar, init_rows, iters: int):
    """Two-level index of a memory ([ASM] hierarchical lookup; the index is built the way the
    memory is, by clustering): the entries qbar [H, K, d] (fp32), rounded to bf16, are clustered
    into C = init_rows.shape[1] groups per head by asm_kmeans (starting from the entries
    init_rows[h]); the first-level centroids are the groups' means; each group lists its
    entries in increasing order. Returns (qhat [H, C, d], offsets [H, C + 1], members [H, K],
    idx [K, H])."""
    qb = np.asarray(qbar, np.float32)
    H, K, d = qb.shape
    bits = qb.view(np.uint32)
    rounded = ((bits + (((bits >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)   # nearest, ties even
    q = np.ascontiguousarray(rounded.transpose(1, 0, 2))                           # [K, H, d]
    idx, cent = asm_kmeans(q, init_rows, iters)
    C = np.asarray(init_rows).shape[1]
    offsets = np.zeros((H, C + 1), np.int32)
    members = np.zeros((H, K), np.int32)
    for h in range(H):
        order = [np.nonzero(idx[:, h] == c)[0] for c in range(C)]
        offsets[h, 1:] = np.cumsum([len(o) for o in order])
        members[h] = np.concatenate(order).astype(np.int32)
    return cent, offsets, members, idx


def group_rows(x, G: int):
    """Calibration rows of a grouped table: x [M, H, ...] -> [M * G, H // G, ...], row (i, h)
    going to table h // G ([ASM] GQA extension: the group's queries are aggregated)."""
    x = np.asarray(x)
    M, H = x.shape[:2]
    y = x.reshape((M, H // G, G) + x.shape[2:])
    y = np.moveaxis(y, 2, 1)                       # [M, G, H // G, ...]
    return np.ascontiguousarray(y.reshape((M * G, H // G) + x.shape[2:]))


def expand_tables(t, G: int):
    """Per-head view of grouped tables: t [H // G, ...] -> [H, ...], head h reading table h // G."""
    return np.repeat(np.asarray(t), G, axis=0)
