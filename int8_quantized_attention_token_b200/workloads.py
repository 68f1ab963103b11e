"""Seeded synthetic inputs for the attention forward pass.

This module only draws random numbers: it holds none of the method's
arithmetic, and it is the one module that both the CUDA path's callers and the
CPU oracle's callers share.

Recipe (the same for every config): a CPU ``torch.Generator`` seeded with
``seed`` draws Q, then K, then V as float32 ``randn(B, H, L, d)``; optional
structure is applied in float32; the result is rounded to fp16.

* ``outliers=True`` (activation outliers, to stress per-token scales):
  ``max(1, round(0.01 d))`` head-dim channels drawn with ``randperm(d)`` are
  multiplied by 20 in Q and K (same channels for every batch and head), then
  for each batch ``max(1, round(0.001 L))`` token positions of Q, and then of
  K, drawn with ``randperm(L)``, are multiplied by 8 (same positions for every
  head).  V stays N(0, 1).
* ``scale`` multiplies all three tensors before the fp16 rounding.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    causal: bool
    outliers: bool = False
    scale: float = 1.0
    seed: int = 0

    @property
    def ops(self) -> float:
        """Algorithmic INT8 ops: 2 B H L^2 d for Q K^T plus the same for P V,
        halved when causal."""
        ops = 4.0 * self.B * self.H * self.L * self.L * self.d
        return ops / 2 if self.causal else ops

    def as_dict(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "L": self.L, "d": self.d,
                "causal": self.causal, "outliers": self.outliers, "scale": self.scale,
                "seed": self.seed}


# The five synthetic configurations of the attention forward pass.
WORKLOADS = [
    Workload("attn_B1_H1_L128_d64", 1, 1, 128, 64, False),
    Workload("attn_B1_H16_L1024_d64", 1, 16, 1024, 64, False),
    Workload("attn_B4_H32_L4096_d128_causal", 4, 32, 4096, 128, True),
    Workload("attn_B2_H32_L4096_d128_causal_outliers", 2, 32, 4096, 128, True, outliers=True),
    Workload("attn_B1_H32_L16384_d128_causal_x0.5", 1, 32, 16384, 128, True, scale=0.5),
]


def by_name(name: str) -> Workload:
    for w in WORKLOADS:
        if w.name == name:
            return w
    raise KeyError(name)


def make_qkv(B: int, H: int, L: int, d: int, seed: int = 0, outliers: bool = False,
             scale: float = 1.0):
    """Return fp16 CPU tensors Q, K, V of shape [B, H, L, d] (see module doc)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    Q = torch.randn(B, H, L, d, dtype=torch.float32, generator=g)
    K = torch.randn(B, H, L, d, dtype=torch.float32, generator=g)
    V = torch.randn(B, H, L, d, dtype=torch.float32, generator=g)
    if outliers:
        n_ch = max(1, round(0.01 * d))
        ch = torch.randperm(d, generator=g)[:n_ch]
        n_tok = max(1, round(0.001 * L))
        q_tok = [torch.randperm(L, generator=g)[:n_tok] for _ in range(B)]
        k_tok = [torch.randperm(L, generator=g)[:n_tok] for _ in range(B)]
        Q[..., ch] *= 20.0
        K[..., ch] *= 20.0
        for b in range(B):
            Q[b, :, q_tok[b], :] *= 8.0
            K[b, :, k_tok[b], :] *= 8.0
    if scale != 1.0:
        Q *= scale
        K *= scale
        V *= scale
    return Q.half(), K.half(), V.half()


def make_workload(w: Workload):
    return make_qkv(w.B, w.H, w.L, w.d, seed=w.seed, outliers=w.outliers, scale=w.scale)
