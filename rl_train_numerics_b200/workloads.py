"""Seeded synthetic inputs for the CPR Gated DeltaNet layer.

This module only draws random inputs; it contains none of the layer's
arithmetic, and both the CUDA path's tests/benchmark and the CPU oracle take
their inputs from it.  The pages measure the layer on three shapes
("NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
section "Solving the linear-attention headache", per-layer table): trainer
forward+backward over 10240 tokens, rollout prefill of 5 x 2048 tokens and
rollout decode of 256 x 1 tokens.  No dataset or trained weights are used;
these draws stand in for the activations of such a layer:

* q, k : N(0,1) per element, L2-normalised over the key dimension of each
         (token, head) in fp32, then rounded to the input dtype (bf16 RNE or
         kept fp32).
* v    : N(0,1), rounded to the input dtype.
* beta : sigmoid(N(0,1)), fp32.
* g    : log-decay, fp32.  ``"softplus"``: g = -softplus(N(0,1)).
         ``"stress"``: g = max(-softplus(N(0, 2.5^2)), -8), then 1 % of the
         entries forced to -8 and 1 % to -1e-7 (long-decay and no-decay tails).

Random numbers come from ``torch.Generator(device).manual_seed(seed)``; the
stream depends on the device type (CPU and CUDA generators differ), so a test
draws once and hands the same tensors to both implementations.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch


@dataclass
class Batch:
    """Packed varlen inputs: q,k [T,H,dk]; v [T,H,dv]; beta,g [T,H]; cu_seqlens [N+1]."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    beta: torch.Tensor
    g: torch.Tensor
    cu_seqlens: torch.Tensor
    lengths: List[int]

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))

    @property
    def n_seqs(self) -> int:
        return len(self.lengths)

    def to(self, device) -> "Batch":
        return Batch(self.q.to(device), self.k.to(device), self.v.to(device),
                     self.beta.to(device), self.g.to(device), self.cu_seqlens.to(device),
                     list(self.lengths))

    def select(self, order: Sequence[int]) -> "Batch":
        """Repack the sequences in ``order`` (a permutation or subset)."""
        cu = [0]
        for n in range(len(self.lengths)):
            cu.append(cu[-1] + self.lengths[n])
        idx = torch.cat([torch.arange(cu[n], cu[n + 1]) for n in order]) if order else \
            torch.zeros(0, dtype=torch.long)
        idx = idx.to(self.q.device)
        lengths = [self.lengths[n] for n in order]
        return Batch(self.q[idx], self.k[idx], self.v[idx], self.beta[idx], self.g[idx],
                     cu_seqlens_of(lengths, self.cu_seqlens.device), lengths)


def cu_seqlens_of(lengths: Sequence[int], device="cpu") -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def _normal(gen, shape, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def draw_tokens(T: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16, seed: int = 0,
                g_mode: str = "softplus", device="cpu"):
    """Draw q,k,v,beta,g for T tokens (see the module docstring for the recipe)."""
    gen = torch.Generator(device=device).manual_seed(int(seed))
    q = _unit_rows(_normal(gen, (T, H, dk), device)).to(dtype)
    k = _unit_rows(_normal(gen, (T, H, dk), device)).to(dtype)
    v = _normal(gen, (T, H, dv), device).to(dtype)
    beta = torch.sigmoid(_normal(gen, (T, H), device))
    if g_mode == "softplus":
        g = -torch.nn.functional.softplus(_normal(gen, (T, H), device))
    elif g_mode == "stress":
        g = torch.clamp(-torch.nn.functional.softplus(2.5 * _normal(gen, (T, H), device)), min=-8.0)
        u = torch.rand((T, H), generator=gen, device=device)
        g = torch.where(u < 0.01, torch.full_like(g, -8.0), g)
        g = torch.where((u >= 0.01) & (u < 0.02), torch.full_like(g, -1e-7), g)
    else:
        raise ValueError(f"unknown g_mode {g_mode!r}")
    return q, k, v, beta.contiguous(), g.contiguous()


def make_batch(lengths: Sequence[int], H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
               seed: int = 0, g_mode: str = "softplus", device="cpu") -> Batch:
    lengths = [int(L) for L in lengths]
    q, k, v, beta, g = draw_tokens(sum(lengths), H, dk, dv, dtype=dtype, seed=seed,
                                   g_mode=g_mode, device=device)
    return Batch(q, k, v, beta, g, cu_seqlens_of(lengths, device), lengths)


# ---------------------------------------------------------------------------
# The five workload shapes
# ---------------------------------------------------------------------------

CHUNK = 64


def tiny(device="cpu") -> Batch:
    """1 sequence, T=256, H=2, d_k=d_v=64, fp32 inputs, seed 0."""
    return make_batch([256], 2, 64, 64, dtype=torch.float32, seed=0, device=device)


def prefill(device="cpu", seed: int = 0) -> Batch:
    """Rollout prefill: 5 x 2048 packed, H=16, d=128, bf16 q/k/v."""
    return make_batch([2048] * 5, 16, 128, 128, dtype=torch.bfloat16, seed=seed, device=device)


def trainer_lengths(total: int = 10240, n_docs: int = 5, min_len: int = 256, seed: int = 3):
    """Document lengths: min_len + Dirichlet(1,...,1) share of the rest, rounded down,
    remainder to the last document."""
    gen = torch.Generator().manual_seed(int(seed))
    e = -torch.log(torch.rand(n_docs, generator=gen, dtype=torch.float64))
    w = e / e.sum()
    spare = total - n_docs * min_len
    lens = [min_len + int(math.floor(float(x) * spare)) for x in w]
    lens[-1] += total - sum(lens)
    return lens


def trainer(device="cpu", seed: int = 0) -> Batch:
    """Trainer forward: 10240 tokens as 5 documents, H=16, d=128, bf16."""
    return make_batch(trainer_lengths(), 16, 128, 128, dtype=torch.bfloat16, seed=seed,
                      device=device)


def decode_prefix_lengths(n_slots: int = 256, lo: int = 1, hi: int = 2047, seed: int = 1):
    gen = torch.Generator().manual_seed(int(seed))
    return [int(x) for x in torch.randint(lo, hi + 1, (n_slots,), generator=gen)]


def decode_tokens(n_steps: int, B: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
                  seed: int = 2, g_mode: str = "softplus", device="cpu"):
    """Fresh tokens for n_steps batched decode steps: tensors [n_steps, B, H, ...]."""
    q, k, v, beta, g = draw_tokens(n_steps * B, H, dk, dv, dtype=dtype, seed=seed,
                                   g_mode=g_mode, device=device)
    return (q.view(n_steps, B, H, dk), k.view(n_steps, B, H, dk), v.view(n_steps, B, H, dv),
            beta.view(n_steps, B, H), g.view(n_steps, B, H))


def stress_lengths(n: int = 64, lo: int = 1, hi: int = 8192, seed: int = 4):
    """Log-uniform lengths in [lo, hi] (the seeded draw is used as is)."""
    gen = torch.Generator().manual_seed(int(seed))
    u = torch.rand(n, generator=gen, dtype=torch.float64)
    return [int(min(hi, max(lo, round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo)))))))
            for x in u]


def stress(device="cpu", n: int = 64, H: int = 32, seed: int = 0) -> Batch:
    """Batch-invariance stress: 64 ragged sequences, H=32, d=128, bf16, stress decays."""
    return make_batch(stress_lengths(n), H, 128, 128, dtype=torch.bfloat16, seed=seed,
                      g_mode="stress", device=device)
