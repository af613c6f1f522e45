"""Independent references used to pin the oracle: library routines, not the oracle's code.

- attention: torch.nn.functional.scaled_dot_product_attention in float64 on the CPU,
  with the retention bias passed as an additive float mask, and torch.logsumexp
  for ln Z;
- cosine: sklearn.metrics.pairwise.cosine_similarity;
- slot removal: numpy.delete.
"""
from __future__ import annotations

import numpy as np
import torch

from memory_bounded_kv_b200.synth import bf16_bits_to_f32


def f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def sdpa_state(q, k, v, scale, bias=None):
    """Attention of each query row over one key set.

    q [R, d]; k, v [n, d]; bias [R, n] or [n] (additive logit terms) or None; all float64.
    Returns (o [R, d], lse [R]) with lse = ln sum exp(logit)."""
    qt = torch.from_numpy(np.asarray(q, np.float64))[None, :, None, :]      # [1, R, 1, d]
    R = qt.shape[1]
    kt = torch.from_numpy(np.asarray(k, np.float64))[None, None].expand(1, R, -1, -1)
    vt = torch.from_numpy(np.asarray(v, np.float64))[None, None].expand(1, R, -1, -1)
    mask = None
    if bias is not None:
        bt = torch.from_numpy(np.asarray(bias, np.float64))
        if bt.dim() == 1:
            bt = bt[None].expand(R, -1)
        mask = bt[None, :, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    logits = torch.matmul(qt, kt.transpose(-1, -2)) * scale
    if mask is not None:
        logits = logits + mask
    lse = torch.logsumexp(logits, dim=-1)
    return o[0, :, 0].numpy(), lse[0, :, 0].numpy()


def cosine_matrix(a, b):
    from sklearn.metrics.pairwise import cosine_similarity
    return cosine_similarity(np.asarray(a, np.float64), np.asarray(b, np.float64))
