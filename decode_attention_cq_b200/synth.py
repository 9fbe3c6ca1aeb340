"""Seeded synthetic decode workloads shaped like InternVL-2.5 visual KV caches.

This module only draws random numbers; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle may consume its tensors.

Recipe (the pages evaluate on real images and video; no dataset or checkpoint
is used here, these caches stand in for them):

* every K and V element is N(0,1) * lambda_c + mu_c, where per (kv-head,
  channel) lambda_c ~ LogNormal(0, 0.5) and mu_c ~ U[-2, 2], drawn separately
  for K and V and shared by every sequence in the batch;
* ``outliers`` channels per kv-head (a seeded random subset) get lambda * 10,
  mimicking the outlier channels of real key caches;
* queries are N(0,1).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One decode-attention workload (a single layer unless ``layers`` > 1)."""

    name: str
    batch: int
    hq: int
    hkv: int
    n: int
    d: int = 128
    dtype: str = "f16"  # storage / compute dtype of q, K, V: "f16" or "f32"
    bits: tuple = (1,)
    outliers: int = 4
    seed: int = 0
    layers: int = 1
    budgets_gb: tuple = field(default_factory=tuple)


WORKLOADS = {
    # tiny single-head case that the oracle finishes in well under a second
    "tiny_n256": Workload("tiny_n256", 1, 1, 1, 256, dtype="f32", bits=(1, 2), outliers=0, seed=0),
    # InternVL-2.5-8B layer shape: 32 query heads, 8 kv-heads, d=128
    "internvl8b_n3328_b16": Workload("internvl8b_n3328_b16", 16, 32, 8, 3328, bits=(1,), seed=1),
    "internvl8b_n8192_b64": Workload("internvl8b_n8192_b64", 64, 32, 8, 8192, bits=(1,), seed=2),
    "bitsweep_n8192_b16": Workload("bitsweep_n8192_b16", 16, 32, 8, 8192, bits=(1, 2, 4, 8), seed=3),
    "budget_n3328_32layers": Workload("budget_n3328_32layers", 0, 32, 8, 3328, bits=(1,), seed=4,
                                      layers=32, budgets_gb=(5, 10, 20, 30)),
}


def torch_dtype(dtype: str) -> torch.dtype:
    return {"f16": torch.float16, "f32": torch.float32}[dtype]


def make_cache(batch: int, hkv: int, n: int, d: int, dtype: str, outliers: int,
               gen: torch.Generator, device) -> torch.Tensor:
    """One cache tensor [batch, hkv, n, d] following the recipe above."""
    lam = torch.exp(0.5 * torch.randn(hkv, d, generator=gen, device=device))
    mu = torch.rand(hkv, d, generator=gen, device=device) * 4.0 - 2.0
    if outliers:
        for h in range(hkv):
            idx = torch.randperm(d, generator=gen, device=device)[:outliers]
            lam[h, idx] *= 10.0
    out = torch.empty(batch, hkv, n, d, dtype=torch_dtype(dtype), device=device)
    for b in range(batch):  # one sequence at a time keeps the fp32 temporary small
        z = torch.randn(hkv, n, d, generator=gen, device=device)
        out[b] = (z * lam[:, None, :] + mu[:, None, :]).to(out.dtype)
    return out


def make_case(batch: int, hq: int, hkv: int, n: int, d: int = 128, dtype: str = "f16",
              outliers: int = 4, seed: int = 0, device="cpu"):
    """q [batch, hq, d], k and v [batch, hkv, n, d] on ``device``, seeded."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    k = make_cache(batch, hkv, n, d, dtype, outliers, gen, device)
    v = make_cache(batch, hkv, n, d, dtype, outliers, gen, device)
    q = torch.randn(batch, hq, d, generator=gen, device=device).to(torch_dtype(dtype))
    return q, k, v


def make_workload(w: Workload, device="cpu", batch: int | None = None, n: int | None = None):
    """Tensors for a named workload (optionally with a smaller batch or n)."""
    return make_case(w.batch if batch is None else batch, w.hq, w.hkv, w.n if n is None else n,
                     w.d, w.dtype, w.outliers, w.seed, device)
