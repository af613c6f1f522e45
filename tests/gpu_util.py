"""Helpers of the GPU parity tests: host <-> device copies and the tolerance checks.

Tolerances (bf16 inputs, fp32 accumulation on the GPU, float64 oracle):
  o:   max-abs <= 2e-2 and rel-L2 <= 1e-3 (over the compared tensor)
  lse: |delta| <= max(1e-4, 2^-22 |lse|), and -inf exactly where the oracle has -inf.
       1e-4 absolute is the target; a float32 lse cannot hold it when |lse| > 419
       (its spacing there reaches 2^-23 |lse| ~ 5e-5 per rounding), so the bound
       becomes two float32 roundings at the magnitude of lse.
Indices, victims, lengths and cache bytes: bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAXABS = 2e-2
O_RELL2 = 1e-3
LSE_ABS = 1e-4
LSE_REL_F32 = 2.0 ** -22


def dev(a: np.ndarray) -> torch.Tensor:
    """Host array -> CUDA tensor (uint16 bit patterns become bfloat16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (ties to even), as float64."""
    f = torch.from_numpy(np.ascontiguousarray(x, np.float64)).to(torch.float32).to(torch.bfloat16)
    return f.to(torch.float64).numpy()


def assert_state_close(o, lse, o_ref, lse_ref, what: str = ""):
    o = np.asarray(o, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    assert o.shape == o_ref.shape, (what, o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - o_ref)
    maxabs = float(err.max()) if err.size else 0.0
    nref = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o - o_ref) / nref) if nref > 0 else float(np.linalg.norm(o))
    assert maxabs <= O_MAXABS, f"{what}: max-abs {maxabs:.3e}"
    assert rel <= O_RELL2, f"{what}: rel-L2 {rel:.3e}"
    if lse is not None:
        lse = np.asarray(lse, np.float64)
        lse_ref = np.asarray(lse_ref, np.float64)
        inf_ref = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse), inf_ref), f"{what}: -inf pattern of lse differs"
        d = np.abs(lse[~inf_ref] - lse_ref[~inf_ref])
        tol = np.maximum(LSE_ABS, LSE_REL_F32 * np.abs(lse_ref[~inf_ref]))
        worst = float((d / tol).max()) if d.size else 0.0
        assert worst <= 1.0, f"{what}: lse |delta| {float(d.max()):.3e} exceeds its bound ({worst:.2f}x)"
    return maxabs, rel


def assert_splits_close(o_part, lse_part, o_ref, lse_ref, what: str = "splits"):
    """Per-split states: lse everywhere; o only where the split is not empty (an empty split's
    o row is not written by the library)."""
    o_part = np.asarray(o_part, np.float64).copy()
    empty = np.isneginf(np.asarray(lse_ref))
    o_part[empty] = 0.0
    return assert_state_close(o_part, lse_part, o_ref, lse_ref, what)


class GpuCache:
    """Device copy of a host cache dict {k, v, log_beta, pos, len}."""

    def __init__(self, k, v, log_beta, pos, len_):
        self.k, self.v = dev(k), dev(v)
        self.log_beta = None if log_beta is None else dev(log_beta)
        self.pos, self.len = dev(pos), dev(len_)

    def to_host(self):
        return dict(k=host(self.k), v=host(self.v), log_beta=None if self.log_beta is None else host(self.log_beta),
                    pos=host(self.pos), len=host(self.len))
