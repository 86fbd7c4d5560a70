"""Seeded synthetic workloads for the MoE expert layer (shared by the oracle side and the GPU side).

This module only draws random inputs. It holds none of the layer's arithmetic: no routing, no
permutation, no expert MLP. It is the one piece both the CPU oracle tests and the CUDA path may use.

Workloads (sizes and value distributions follow the benchmark descriptions of "Olmo-core 3" on
unite.ai, section "Benchmark da trilioni di parametri": random routing is what the system benchmarks
used, and "Parallelismo, precisione e tecniche di memoria": the MXFP8 comparison ran with work spread
uniformly over experts):

  tiny       T=256   d=128  F=256  E=8   k=2  fp32, learned router
  e8_bf16    T=8192  d=2048 F=1024 E=8   k=4  bf16, learned router
  e128_bf16  T=8192  d=2048 F=1024 E=128 k=4  bf16, uniform random routing (given as input)
  e128_skew  T=16384 d=2048 F=1024 E=128 k=4  bf16, learned router + Zipf-like bias 1.2*ln(1/rank)
  e128_mxfp8 T=16384 d=4096 F=1536 E=128 k=4  MXFP8 operands, uniform random routing

Recipe (every draw from one torch.Generator seeded with `seed`, in this order):
  x ~ N(0,1) [T,d]; W_r ~ N(0,0.02) [E,d]; W13 ~ N(0,0.02) [E,2F,d] (rows 0..F-1 gate, F..2F-1 up);
  W2 ~ N(0,0.02) [E,d,F]; dout ~ N(0,1) [T,d]; then, for uniform routing, u ~ U(0,1) [T,E] whose
  k smallest-ranked columns (argsort ascending, first k) are the token's experts, and scores
  s ~ N(0,1) [T,k]. For uniform routing the gates are the config's own recipe: softmax over the k
  scores, computed here in fp64 and stored as fp32.
Values are drawn in fp32 and rounded to the storage dtype (round-to-nearest-even for bf16); both the
oracle and the GPU consume exactly the rounded values.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    F: int
    E: int
    k: int
    dtype: str          # "fp32" | "bf16" | "mxfp8"
    routing: str        # "learned" | "uniform"
    skew: float = 0.0   # Zipf-like bias strength (learned routing only)
    renorm: bool = True

    @property
    def storage_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 256, 128, 256, 8, 2, "fp32", "learned"),
    "e8_bf16": Workload("e8_bf16", 8192, 2048, 1024, 8, 4, "bf16", "learned"),
    "e128_bf16": Workload("e128_bf16", 8192, 2048, 1024, 128, 4, "bf16", "uniform"),
    "e128_skew": Workload("e128_skew", 16384, 2048, 1024, 128, 4, "bf16", "learned", skew=1.2),
    "e128_mxfp8": Workload("e128_mxfp8", 16384, 4096, 1536, 128, 4, "mxfp8", "uniform"),
    # the MXFP8 workload's shapes in bf16, for the bf16 vs MXFP8 comparison
    "e128_bf16_wide": Workload("e128_bf16_wide", 16384, 4096, 1536, 128, 4, "bf16", "uniform"),
}


def skew_bias(E: int, strength: float) -> torch.Tensor:
    """Per-expert additive logit bias strength*ln(1/rank), rank = e+1 (fp32). Input recipe only."""
    r = torch.arange(1, E + 1, dtype=torch.float64)
    return (strength * torch.log(1.0 / r)).to(torch.float32)


def _normal(g, shape, std, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def make_inputs(w: Workload, seed: int = 0, device: str = "cpu") -> dict:
    """Draw every input of one layer call (fwd + bwd) for workload `w`.

    Returns a dict of tensors on `device` in their storage dtype:
      x[T,d], W_r[E,d], W13[E,2F,d], W2[E,d,F], dout[T,d], bias[E] (fp32 or None),
      and for uniform routing idx[T,k] int32 + gates[T,k] fp32 (else None).
    """
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    sd = w.storage_dtype
    T, d, F, E, k = w.T, w.d, w.F, w.E, w.k
    out = {}
    out["x"] = _normal(g, (T, d), 1.0, device).to(sd)
    out["W_r"] = _normal(g, (E, d), 0.02, device).to(sd)
    out["W13"] = _normal(g, (E, 2 * F, d), 0.02, device).to(sd)
    out["W2"] = _normal(g, (E, d, F), 0.02, device).to(sd)
    out["dout"] = _normal(g, (T, d), 1.0, device).to(sd)
    out["bias"] = skew_bias(E, w.skew).to(device) if (w.routing == "learned" and w.skew) else None
    if w.routing == "uniform":
        u = torch.rand((T, E), generator=g, device=device, dtype=torch.float32)
        idx = torch.argsort(u, dim=1, stable=True)[:, :k].to(torch.int32)
        s = torch.randn((T, k), generator=g, device=device, dtype=torch.float32)
        gates = torch.softmax(s.double(), dim=1).to(torch.float32)
        out["idx"], out["gates"] = idx.contiguous(), gates.contiguous()
    else:
        out["idx"], out["gates"] = None, None
    return out


def max_padded_rows(T: int, k: int, E: int, align: int = 32) -> int:
    """Upper bound on routed rows once every expert's group start is aligned to `align` rows."""
    return T * k + (align - 1) * E


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Workload", "WORKLOADS", "make_inputs", "skew_bias", "max_padded_rows", "ceil_div"]
