"""Seeded synthetic inputs shaped like the last-layer Q/K/V projections the
LinearARD method distils.

This module only draws and shapes input tensors; it holds none of the
relation-KL arithmetic.  Both the CUDA path and the CPU oracle are fed from
it, the oracle with the same (already rounded) values converted to float64.

Recipe (stands in for LLaMA2-7B / LLaMA3-8B / Mistral-7B last-layer
projections on PG19 text, which are not available here; only their shapes
are used):

* Q and K relations: X_pre ~ N(0, 1) of shape [B, H, n, d].  Teacher
  X_t = RoPE(X_pre, theta, p); student X_s = RoPE(X_pre + 0.05 N(0, 1), theta,
  p * s) with p = 0..n-1 and s the position-interpolation factor (1/8 or 1/4,
  the PI 8x / 4x student of the LinearARD notes, "实验关键数据 / 主实验").
* V relation: V_t ~ N(0, 1); V_s = V_t + 0.05 N(0, 1); no rotation.
* Self-relations: Y = X for every relation (LinearARD notes, 关键设计 1).
* RoPE follows the common "rotate-half" convention: pairs (k, k + d/2) turn
  by angle p * theta^(-2k/d).  The pages give no formula; this is the
  plainest reading.  Angles are formed in float64, applied in float32.
* Rounding: float32 values are rounded to bfloat16 (round-to-nearest-even)
  for the bf16 workloads; the fp32 workload keeps float32.
* Each (workload seed, relation, tensor) draws from its own generator.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Tuple

import torch

RELATIONS = ("Q", "K", "V")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: Dict[str, int]  # relation -> number of heads
    n: int
    d: int
    dtype: str  # "bf16" or "fp32"
    theta: float
    pi_scale: float
    seed: int
    causal: bool = True

    @property
    def relations(self) -> Tuple[str, ...]:
        return tuple(r for r in RELATIONS if r in self.heads)

    @property
    def tau(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def causal_logits(self) -> int:
        """Causal logits of one fwd+bwd pass over every relation: sum B*H*n(n+1)/2."""
        per = self.n * (self.n + 1) // 2 if self.causal else self.n * self.n
        return sum(self.B * h * per for h in self.heads.values())

    def algorithmic_flops(self) -> int:
        """12*d flop per logit: 2 GEMMs in the LSE pass, 4 in the gradient pass."""
        return 12 * self.d * self.causal_logits()


# The five workloads: a small fp32 case, and bf16 cases at the LLaMA2-7B
# native context, 16K, 32K, and a GQA shape with a ragged tail.
WORKLOADS = {
    "fp32-small": Workload("qq-self-relation B1 H2 n256 d64 fp32", 1, {"Q": 2}, 256, 64, "fp32",
                           1e4, 1 / 8, 0),
    "n4096": Workload("qkv-self-relation B1 H32 n4096 d128 bf16", 1, {"Q": 32, "K": 32, "V": 32},
                      4096, 128, "bf16", 1e4, 1 / 8, 1),
    "n16384": Workload("qkv-self-relation B1 H32 n16384 d128 bf16", 1,
                       {"Q": 32, "K": 32, "V": 32}, 16384, 128, "bf16", 1e4, 1 / 4, 2),
    "n32768": Workload("qkv-self-relation B1 H32 n32768 d128 bf16", 1,
                       {"Q": 32, "K": 32, "V": 32}, 32768, 128, "bf16", 1e4, 1 / 8, 3),
    "gqa-n8000": Workload("qkv-self-relation GQA B2 Hq32 Hkv8 n8000 d128 bf16", 2,
                          {"Q": 32, "K": 8, "V": 8}, 8000, 128, "bf16", 5e5, 1 / 4, 4),
}


def custom(B: int, H: int, n: int, d: int, dtype: str = "bf16", seed: int = 0,
           relations=RELATIONS, theta: float = 1e4, pi_scale: float = 1 / 8,
           causal: bool = True) -> Workload:
    """A workload of arbitrary size with the same recipe (used for parity sweeps)."""
    return Workload(f"custom B{B} H{H} n{n} d{d} {dtype}", B, {r: H for r in relations}, n, d,
                    dtype, theta, pi_scale, seed, causal)


def _gen(seed: int, rel: str, tensor: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(1_000_003 * (seed + 1) + 101 * (RELATIONS.index(rel) + 1) + tensor)
    return g


def rope(x: torch.Tensor, positions: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half RoPE of x [..., n, d] at (possibly fractional) positions [n]."""
    d = x.shape[-1]
    half = d // 2
    k = torch.arange(half, dtype=torch.float64)
    inv_freq = theta ** (-2.0 * k / d)
    ang = positions.to(torch.float64)[:, None] * inv_freq[None, :]
    cos = torch.cos(ang).to(torch.float32)
    sin = torch.sin(ang).to(torch.float32)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat((x1 * cos - x2 * sin, x1 * sin + x2 * cos), dim=-1)


def _round(x: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    if dtype == "fp32":
        return x.to(torch.float32)
    raise ValueError(f"unknown dtype {dtype}")


def make_relation(w: Workload, rel: str) -> Tuple[torch.Tensor, torch.Tensor]:
    """Teacher and student projections (X_t, X_s) of one relation, CPU tensors
    [B, H_rel, n, d] in the workload's dtype.  Y = X (self-relation)."""
    H = w.heads[rel]
    shape = (w.B, H, w.n, w.d)
    base = torch.randn(shape, generator=_gen(w.seed, rel, 0), dtype=torch.float32)
    noise = torch.randn(shape, generator=_gen(w.seed, rel, 1), dtype=torch.float32)
    if rel in ("Q", "K"):
        p = torch.arange(w.n, dtype=torch.float64)
        xt = rope(base, p, w.theta)
        xs = rope(base + 0.05 * noise, p * w.pi_scale, w.theta)
    else:
        xt = base
        xs = base + 0.05 * noise
    return _round(xt, w.dtype).contiguous(), _round(xs, w.dtype).contiguous()


def make_all(w: Workload) -> Dict[str, Tuple[torch.Tensor, torch.Tensor]]:
    return {rel: make_relation(w, rel) for rel in w.relations}


def as_f64(t: torch.Tensor):
    """Exact float64 copy (numpy) of a bf16/fp32 tensor, for the oracle."""
    return t.detach().to("cpu").to(torch.float64).numpy()
