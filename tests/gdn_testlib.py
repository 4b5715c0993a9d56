"""Helpers shared by the GPU tests: oracle runs on selected units, error metrics,
guarded (canary) output buffers.

Tolerances (float outputs compared with the fp64 oracle):
  fp32 inputs: max|o - o_ref| <= 1e-5 * RMS(o_ref)
  bf16 inputs: max|o - o_ref| <= 2e-3 * RMS(o_ref)
measured on the library's fp32-output mode (the pre-cast fp32 result); bf16
outputs are checked to be exactly the round-to-nearest-even of that result.
Final states use the same bounds relative to RMS(S_ref).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_F32 = 1e-5
TOL_BF16 = 2e-3
CANARY = 4096  # guard elements on each side of a guarded buffer


def tol_for(dtype) -> float:
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def rms(x) -> float:
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def rel_err(got, ref) -> float:
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref)) / max(rms(ref), 1e-30))


def oracle_unit(batch, n: int, h: int, h0=None, scale: float = 1.0):
    """Oracle over sequence n, head h of a workloads.Batch (CPU tensors)."""
    cu = batch.cu_seqlens.cpu().tolist()
    sl = slice(cu[n], cu[n + 1])
    T = cu[n + 1] - cu[n]
    pick = lambda t: t[sl, h:h + 1].cpu()  # noqa: E731
    h0u = None if h0 is None else h0[n:n + 1, h:h + 1].cpu()
    o, s = oracle.forward(pick(batch.q), pick(batch.k), pick(batch.v),
                          batch.beta[sl, h:h + 1].cpu(), batch.g[sl, h:h + 1].cpu(),
                          np.array([0, T], np.int32), h0=h0u, scale=scale)
    return o[:, 0, :], s[0, 0]


def oracle_prefix_state(batch, n: int, h: int, upto: int, h0=None):
    """Oracle state of sequence n, head h after its first `upto` tokens."""
    cu = batch.cu_seqlens.cpu().tolist()
    sl = slice(cu[n], cu[n] + upto)
    pick = lambda t: t[sl, h:h + 1].cpu()  # noqa: E731
    h0u = None if h0 is None else h0[n:n + 1, h:h + 1].cpu()
    _, s = oracle.forward(pick(batch.q), pick(batch.k), pick(batch.v),
                          batch.beta[sl, h:h + 1].cpu(), batch.g[sl, h:h + 1].cpu(),
                          np.array([0, upto], np.int32), h0=h0u)
    return s[0, 0]


def guarded(shape, dtype, device="cuda"):
    """A tensor view with CANARY NaN-pattern elements before and after it."""
    n = int(np.prod(shape))
    base = torch.full((n + 2 * CANARY,), float("nan"), dtype=dtype, device=device)
    view = base[CANARY:CANARY + n].view(*shape)
    return base, view


def canaries_intact(base) -> bool:
    head, tail = base[:CANARY], base[-CANARY:]
    return bool(torch.isnan(head).all()) and bool(torch.isnan(tail).all())
