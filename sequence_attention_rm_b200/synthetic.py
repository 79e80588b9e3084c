"""Seeded synthetic inputs for the ring-attention workloads.

This module holds only random-number generation and the workload shapes; it
contains none of the attention arithmetic, and both the CUDA path's tests and
the CPU oracle consume exactly the bytes it produces.

Recipe: a torch CPU ``Generator`` seeded with ``1000 * workload_id + role``
(role 0: Q, 1: K, 2: V, 3: dO) draws iid fp32 N(0, 1) values in global token
order [B, N, H, d]; Q/K/V are multiplied by the workload's ``qkv_scale``; the
result is cast to the workload dtype with round-to-nearest-even.  The oracle
upcasts those exact values to fp64.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    """One ring-attention problem (shapes only)."""

    wid: int            # seed base (1000 * wid + role)
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    P: int
    layout: str         # "contiguous" | "zigzag" | "striped"
    causal: bool
    dtype: torch.dtype
    qkv_scale: float = 1.0
    backward: bool = False

    def scaled(self, N: int, **kw) -> "Workload":
        return dataclasses.replace(self, N=N, **kw)

    @property
    def local(self) -> int:
        return self.N // self.P


# The five workloads (tiny fp32 ring; Llama-like zigzag; striped 128k;
# tabular multi-axis; long zigzag + Ulysses repack).
TINY_RING = Workload(1, "tiny-noncausal-ring-fp32", B=1, Hq=2, Hkv=2, N=256, d=64, P=4,
                     layout="contiguous", causal=False, dtype=torch.float32)
LLAMA_ZIGZAG = Workload(2, "llama-causal-zigzag-16k", B=1, Hq=16, Hkv=8, N=16384, d=128, P=2,
                        layout="zigzag", causal=True, dtype=torch.bfloat16, qkv_scale=0.5,
                        backward=True)
STRIPED_128K = Workload(3, "causal-striped-128k", B=1, Hq=16, Hkv=8, N=131072, d=128, P=8,
                        layout="striped", causal=True, dtype=torch.bfloat16, qkv_scale=0.5,
                        backward=True)
LONG_ZIGZAG_256K = Workload(5, "long-causal-zigzag-256k", B=1, Hq=16, Hkv=8, N=262144, d=128, P=8,
                            layout="zigzag", causal=True, dtype=torch.bfloat16, qkv_scale=0.5,
                            backward=True)


@dataclass(frozen=True)
class TabularWorkload:
    """Tabular (batch, rows, features, embed) tensor attended along two axes."""

    wid: int
    name: str
    batch: int
    rows: int
    features: int
    embed: int
    heads: int
    P: int              # ring ranks along the rows axis (contiguous)
    dtype: torch.dtype

    @property
    def head_dim(self) -> int:
        return self.embed // self.heads

    def scaled(self, rows: int) -> "TabularWorkload":
        return dataclasses.replace(self, rows=rows)


TABULAR = TabularWorkload(4, "tabular-multiaxis-150k", batch=1, rows=150000, features=5, embed=96,
                          heads=4, P=8, dtype=torch.bfloat16)

WORKLOADS = {w.wid: w for w in (TINY_RING, LLAMA_ZIGZAG, STRIPED_128K, LONG_ZIGZAG_256K)}


def _draw(wid: int, role: int, shape, scale: float, dtype: torch.dtype) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 * wid + role)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(dtype)


def attention_inputs(w: Workload, with_dout: bool = True):
    """(q, k, v, dout) CPU tensors in global token order [B, N, H, d]."""
    q = _draw(w.wid, 0, (w.B, w.N, w.Hq, w.d), w.qkv_scale, w.dtype)
    k = _draw(w.wid, 1, (w.B, w.N, w.Hkv, w.d), w.qkv_scale, w.dtype)
    v = _draw(w.wid, 2, (w.B, w.N, w.Hkv, w.d), w.qkv_scale, w.dtype)
    dout = _draw(w.wid, 3, (w.B, w.N, w.Hq, w.d), 1.0, w.dtype) if with_dout else None
    return q, k, v, dout


def tabular_inputs(w: TabularWorkload):
    """Three independent (batch, rows, features, embed) tensors: q, k, v."""
    shape = (w.batch, w.rows, w.features, w.embed)
    return tuple(_draw(w.wid, role, shape, 1.0, w.dtype) for role in range(3))


def tensor(seed: int, shape, dtype=torch.float32, scale: float = 1.0) -> torch.Tensor:
    """Generic seeded N(0, scale^2) tensor (for merge / repack / permute cases)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(dtype)
