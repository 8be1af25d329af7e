"""Seeded synthetic workloads for Positional-LSH approximate ALiBi attention.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It holds shapes, seeds and random inputs only -- none of the method's
arithmetic (no hashing, no binning, no attention).

Workloads (all inputs iid N(0,1), drawn from a seeded torch CPU generator in
the order Q, K, V, then cast to the workload dtype):

  single_head_n1024   B=1  H=1  / H_kv=1  n=1024   d=64  fp32 non-causal s=8   seed 0  sigma=16
  mha8_n8192          B=1  H=8  / H_kv=8  n=8192   d=128 bf16 non-causal s=10  seed 1
  qwen3_0p6b_n32k     B=2  H=16 / H_kv=8  n=32768  d=128 bf16 causal     s=20  seed 2
  mistral7b_n16k      B=1  H=32 / H_kv=8  n=16384  d=128 bf16 causal     s in {10,20,40} seed 3
  long_n128k          B=1  H=40 / H_kv=8  n=131072 d=128 bf16 causal     s=16  seed 4

The per-head ALiBi length scale is sigma_h = 1/slope_h with the standard
ALiBi slope schedule slope_h = 2^(-8(h+1)/H), h = 0..H-1.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    H_kv: int
    n: int
    d: int
    dtype: str          # "f32" or "bf16"
    causal: bool
    s: int
    seed: int
    sigma_const: Optional[float] = None   # single-head workload uses a fixed sigma
    oracle_rows: int = 0                  # rows per head the oracle checks (0 = all)

    def sigmas(self) -> List[float]:
        """Per-query-head sigma_h (1/ALiBi slope)."""
        if self.sigma_const is not None:
            return [float(self.sigma_const)] * self.H
        return [2.0 ** (8.0 * (h + 1) / self.H) for h in range(self.H)]

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def query_tokens(self) -> int:
        return self.B * self.n


WORKLOADS = {
    "single_head_n1024": Workload("single_head_n1024", 1, 1, 1, 1024, 64, "f32", False, 8, 0,
                                  sigma_const=16.0),
    "mha8_n8192": Workload("mha8_n8192", 1, 8, 8, 8192, 128, "bf16", False, 10, 1),
    "qwen3_0p6b_n32k": Workload("qwen3_0p6b_n32k", 2, 16, 8, 32768, 128, "bf16", True, 20, 2,
                                oracle_rows=256),
    "mistral7b_n16k": Workload("mistral7b_n16k", 1, 32, 8, 16384, 128, "bf16", True, 20, 3,
                               oracle_rows=256),
    "long_n128k": Workload("long_n128k", 1, 40, 8, 131072, 128, "bf16", True, 16, 4,
                           oracle_rows=512),
}

# The s sweep of the Mistral-7B-shaped workload.
MISTRAL_S_SWEEP = (10, 20, 40)

# The workload the headline throughput is quoted on.
HEADLINE = "qwen3_0p6b_n32k"


def make_qkv(w: Workload, device: str = "cpu") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q [B,H,n,d], K [B,H_kv,n,d], V [B,H_kv,n,d] from torch.Generator().manual_seed(seed).

    Always drawn on the CPU in fp32 (so the oracle and the GPU see the same
    bits), then cast to the workload dtype and moved to `device`.
    """
    g = torch.Generator().manual_seed(w.seed)
    q = torch.randn(w.B, w.H, w.n, w.d, generator=g, dtype=torch.float32)
    k = torch.randn(w.B, w.H_kv, w.n, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(w.B, w.H_kv, w.n, w.d, generator=g, dtype=torch.float32)
    dt = w.torch_dtype
    return q.to(dt).to(device), k.to(dt).to(device), v.to(dt).to(device)


def make_qkv_device(w: Workload, device: str) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Same shapes and distribution as make_qkv, drawn directly on `device`.

    For timing only: the values differ from make_qkv's (a device generator),
    which does not matter to throughput.
    """
    g = torch.Generator(device=device).manual_seed(w.seed)
    dt = w.torch_dtype
    q = torch.randn(w.B, w.H, w.n, w.d, generator=g, device=device, dtype=torch.float32).to(dt)
    k = torch.randn(w.B, w.H_kv, w.n, w.d, generator=g, device=device, dtype=torch.float32).to(dt)
    v = torch.randn(w.B, w.H_kv, w.n, w.d, generator=g, device=device, dtype=torch.float32).to(dt)
    return q, k, v


def sample_rows(n: int, count: int, seed: int) -> List[int]:
    """`count` distinct query rows in [0, n), always including 0 and n-1, from a fixed-seed RNG."""
    if count <= 0 or count >= n:
        return list(range(n))
    g = torch.Generator().manual_seed(1_000_003 + seed)
    perm = torch.randperm(n, generator=g).tolist()
    rows = {0, n - 1}
    for r in perm:
        if len(rows) >= count:
            break
        rows.add(r)
    return sorted(rows)
