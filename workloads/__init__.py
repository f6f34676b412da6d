"""Seeded synthetic workloads for the sharded MLP.

This module holds only the workload table and the seeded input generators.
It contains none of the MLP's arithmetic, and it is the one module that both
the fp64 oracle's callers and the CUDA path's callers share.

Input recipe (one ``torch.Generator('cpu')`` per workload, seeded with the
workload's seed, drawing with ``torch.randn`` in this fixed order):

    X[n, d]          ~ N(0, 1)
    A = W_gate[d, f] ~ N(0, s_in^2)
    W_up[d, f]       ~ N(0, s_in^2)     (gated MLP only)
    B = W_down[f, d] ~ N(0, s_out^2)
    dY[n, d]         ~ N(0, 1)          (backward only)

then cast (round to nearest even) to the workload's dtype.  For the bf16
workloads s_in = s_out = the weight std of the workload (0.02, or 0.015 for
the 70B shape).  For the fp32 GeLU block the weights are N(0, 1/d_in) with
d_in the matrix's fan-in: s_in = 1/sqrt(d_model), s_out = 1/sqrt(d_ff).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    act: str            # "gelu" or "swiglu"
    dtype: str          # "f32" or "bf16"
    n: int              # tokens
    d: int              # d_model
    f: int              # d_ff
    P: int              # logical weight shards
    seed: int
    w_std: float | None  # weight std (None: N(0, 1/fan_in))
    sched: str = "weight_shards"  # or "tsp_ring", "tsp_ring_fused", "fused", "shard_passes"
    backward: bool = False

    def flops_forward(self) -> int:
        """Algorithmic forward FLOPs: 2 GEMMs (GeLU) or 3 GEMMs (SwiGLU)."""
        gemms = 3 if self.act == "swiglu" else 2
        return 2 * gemms * self.n * self.d * self.f

    def flops_backward(self) -> int:
        """Algorithmic backward FLOPs (no recompute): dH, dX(2), dWg, dWu, dWd for
        SwiGLU (6 GEMMs); dH, dX, dA, dB for GeLU (4 GEMMs)."""
        gemms = 6 if self.act == "swiglu" else 4
        return 2 * gemms * self.n * self.d * self.f

    def scaled(self, n=None, d=None, f=None, P=None, name=None) -> "Workload":
        return dataclasses.replace(self, n=n or self.n, d=d or self.d, f=f or self.f,
                                   P=P or self.P, name=name or self.name + "_small")


# The five workloads: the fp32 GeLU block, the Llama-3-8B-shaped SwiGLU block,
# the TSP long-context ring, the 70B-shaped block and the fwd+bwd of the
# Llama-3-8B-shaped block.
WORKLOADS = {
    "gelu_f32_n64_d128_f512": Workload("gelu_f32_n64_d128_f512", "gelu", "f32", 64, 128, 512, 2,
                                       seed=0, w_std=None),
    "swiglu_bf16_n4096_d4096_f14336": Workload("swiglu_bf16_n4096_d4096_f14336", "swiglu", "bf16",
                                               4096, 4096, 14336, 8, seed=1, w_std=0.02),
    "tsp_ring_bf16_n32768_d4096_f14336": Workload("tsp_ring_bf16_n32768_d4096_f14336", "swiglu",
                                                  "bf16", 32768, 4096, 14336, 8, seed=2,
                                                  w_std=0.02, sched="tsp_ring"),
    "swiglu_bf16_n8192_d8192_f28672": Workload("swiglu_bf16_n8192_d8192_f28672", "swiglu", "bf16",
                                               8192, 8192, 28672, 8, seed=3, w_std=0.015),
    "swiglu_bf16_fwdbwd_n4096_d4096_f14336": Workload("swiglu_bf16_fwdbwd_n4096_d4096_f14336",
                                                      "swiglu", "bf16", 4096, 4096, 14336, 8,
                                                      seed=4, w_std=0.02, backward=True),
}

GELU_F32 = WORKLOADS["gelu_f32_n64_d128_f512"]
LLAMA8B = WORKLOADS["swiglu_bf16_n4096_d4096_f14336"]
TSP_RING = WORKLOADS["tsp_ring_bf16_n32768_d4096_f14336"]
LLAMA70B = WORKLOADS["swiglu_bf16_n8192_d8192_f28672"]
FWD_BWD = WORKLOADS["swiglu_bf16_fwdbwd_n4096_d4096_f14336"]


def torch_dtype(wl: Workload) -> torch.dtype:
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def make_inputs(wl: Workload, seed: int | None = None, backward: bool | None = None) -> dict:
    """Seeded CPU tensors of the workload's shapes and dtype.

    Returns a dict with keys X, A (= W_gate), Wu (None for GeLU), B (= W_down)
    and dY (None unless backward).
    """
    seed = wl.seed if seed is None else seed
    backward = wl.backward if backward is None else backward
    g = torch.Generator("cpu").manual_seed(seed)
    if wl.w_std is None:
        s_in, s_out = 1.0 / math.sqrt(wl.d), 1.0 / math.sqrt(wl.f)
    else:
        s_in = s_out = wl.w_std
    dt = torch_dtype(wl)
    X = torch.randn(wl.n, wl.d, generator=g)
    A = torch.randn(wl.d, wl.f, generator=g).mul_(s_in)
    Wu = torch.randn(wl.d, wl.f, generator=g).mul_(s_in) if wl.act == "swiglu" else None
    B = torch.randn(wl.f, wl.d, generator=g).mul_(s_out)
    dY = torch.randn(wl.n, wl.d, generator=g) if backward else None
    cast = (lambda t: None if t is None else t.to(dt).contiguous())
    return {"X": cast(X), "A": cast(A), "Wu": cast(Wu), "B": cast(B), "dY": cast(dY)}


def sample_rows(n: int, count: int, seed: int) -> list[int]:
    """Seeded sample of token rows: ``count`` random rows plus the first and last."""
    g = torch.Generator("cpu").manual_seed(seed + 7919)
    k = min(count, n)
    rows = set(torch.randperm(n, generator=g)[:k].tolist())
    rows.update({0, n - 1})
    return sorted(rows)


def cover_rows(n: int, block: int, seed: int, groups=()) -> list[int]:
    """Seeded token rows that touch every launch and tile of a full-size run.

    One seeded row inside every ``block``-row block of [0, n) (a 256-row pair
    tile, say), plus the first and last row of [0, n) and of every
    ``(begin, end)`` half-open range in ``groups`` (row groups, sequence
    shards).  Sorted, without repeats.
    """
    g = torch.Generator("cpu").manual_seed(seed + 104729)
    rows = {0, n - 1}
    for b0 in range(0, n, block):
        size = min(block, n - b0)
        rows.add(b0 + int(torch.randint(size, (1,), generator=g)))
    for b, e in groups:
        rows.update({b, e - 1})
    return sorted(r for r in rows if 0 <= r < n)


def cover_cols(f: int, P: int, block: int, seed: int) -> list[int]:
    """Seeded hidden columns that touch every weight shard and column tile.

    Every shard's first and last column, plus one seeded column inside every
    ``block``-column block of [0, f).  Sorted, without repeats.
    """
    fs = f // P
    cols = set()
    for w in range(P):
        cols.update({w * fs, w * fs + fs - 1})
    cols.update(cover_rows(f, block, seed))
    return sorted(cols)


# ---------------------------------------------------------------------------
# TSP attention


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    """Multi-head self-attention block under the TSP schedule: n tokens in P
    sequence shards, n_heads heads of d / n_heads in P parameter shards."""
    name: str
    n: int              # tokens
    d: int              # d_model
    heads: int
    P: int              # sequence shards = parameter shards
    causal: bool
    seed: int
    w_std: float

    @property
    def dh(self) -> int:
        return self.d // self.heads

    def flops(self) -> dict:
        """Algorithmic FLOPs: the four projections (2 n d^2 each) and the core
        (2 d per query-key pair for the scores and 2 d for the weighted values;
        with the causal mask only the n (n + 1) / 2 visible pairs count)."""
        pairs = self.n * (self.n + 1) // 2 if self.causal else self.n * self.n
        return {"projections": 4 * 2 * self.n * self.d * self.d, "core": 4 * pairs * self.d}


# Input recipe: one torch.Generator('cpu') seeded with the workload's seed,
# torch.randn in the order X[n, d] ~ N(0, 1), W_q, W_k, W_v, W_o [d, d] ~
# N(0, w_std^2), cast (round to nearest even) to bf16.  The long-context shape
# is the TSP ring workload's (32768 tokens in 8 sequence shards of 4096,
# d_model 4096) with Llama-3-8B's 32 heads of 128.
ATTN_WORKLOADS = {
    "tsp_attn_causal_bf16_n32768_d4096_h32": AttnWorkload(
        "tsp_attn_causal_bf16_n32768_d4096_h32", 32768, 4096, 32, 8, True, seed=5, w_std=0.02),
    "tsp_attn_bf16_n32768_d4096_h32": AttnWorkload(
        "tsp_attn_bf16_n32768_d4096_h32", 32768, 4096, 32, 8, False, seed=6, w_std=0.02),
}
TSP_ATTN = ATTN_WORKLOADS["tsp_attn_causal_bf16_n32768_d4096_h32"]


def make_attn_inputs(wl: AttnWorkload, seed: int | None = None) -> dict:
    """Seeded bf16 CPU tensors X, Wq, Wk, Wv, Wo of the workload's shapes."""
    g = torch.Generator("cpu").manual_seed(wl.seed if seed is None else seed)
    X = torch.randn(wl.n, wl.d, generator=g)
    W = [torch.randn(wl.d, wl.d, generator=g).mul_(wl.w_std) for _ in range(4)]
    out = {"X": X}
    out.update(zip(("Wq", "Wk", "Wv", "Wo"), W))
    return {k: v.to(torch.bfloat16).contiguous() for k, v in out.items()}


def make_qkv(n: int, d: int, seed: int, std: float = 1.0) -> dict:
    """Seeded bf16 Q, K, V [n, d] ~ N(0, std^2) for tests of the attention core
    alone (drawn in the order Q, K, V)."""
    g = torch.Generator("cpu").manual_seed(seed)
    return {k: torch.randn(n, d, generator=g).mul_(std).to(torch.bfloat16).contiguous()
            for k in ("Q", "K", "V")}
