"""Seeded synthetic inputs for the SLA2 attention forward pass.

This module holds no arithmetic of the method itself: it only draws tensors.
Both the CUDA path (through the tests and the bench) and the CPU oracle are fed
from here, so the two sides always see the same bytes.

Workloads follow the shapes of the Wan2.1 video-DiT attention calls that the
SLA2 paper evaluates on (SLA2 detail page, section 5 "Experiments", Table 1:
Wan2.1-1.3B-480P and Wan2.1-14B-720P; 12 and 40 heads of width 128). The
activations themselves are not available, so each tensor is

    X = noise ~ N(0, 1)  +  per-(b, h, 64-token block) d-vector offset ~ N(0, var)

with K additionally carrying a per-(b, h) channel bias ~ N(0, 1) (the bias is
what K smoothing removes). Router projections are ~ N(0, 1/d) (variance), one
[d_in, d_out] matrix per head; alpha ~ U(0, 1) per (head, query block).

Draw order (a fixed contract; changing it changes every test input):
Q, K, V noise; Q, K, V block offsets; K channel bias; proj_q; proj_k; alpha.
All draws are fp32 from a CPU ``torch.Generator`` seeded per workload, then
Q/K/V are rounded to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch

BLOCK_Q = 128   # b_q, tokens per query block
BLOCK_K = 64    # b_k, tokens per key block


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    topk_frac: float
    offset_var: float = 0.5
    seed: int = 0
    alpha_one: bool = False   # alpha = 1 everywhere (the dense check at k% = 100)

    @property
    def nq(self) -> int:
        return self.N // BLOCK_Q

    @property
    def nk(self) -> int:
        return self.N // BLOCK_K

    def with_frac(self, frac: float, alpha_one: bool = False) -> "Workload":
        return replace(self, name=f"{self.name}@{frac:g}", topk_frac=frac, alpha_one=alpha_one)


# The five workloads: a small case, the Wan2.1-1.3B-480P attention shape at 97%
# sparsity (the headline), the Wan2.1-14B-720P shape at 95%, a batched d=64 case
# with a more peaked router, and the sparsity sweep on the 1.3B shape.
WORKLOADS = {
    "small": Workload("small", 1, 1, 2048, 64, 0.10, 0.5, 0),
    "wan1.3b": Workload("wan1.3b", 1, 12, 32768, 128, 0.03, 0.5, 1),
    "wan14b": Workload("wan14b", 1, 40, 75776, 128, 0.05, 0.5, 2),
    "batched": Workload("batched", 2, 24, 16384, 64, 0.10, 1.0, 3),
}
SWEEP_FRACS = (0.03, 0.05, 0.10, 0.20, 1.0)


def sweep_workloads():
    base = WORKLOADS["wan1.3b"]
    return [base.with_frac(f, alpha_one=(f == 1.0)) for f in SWEEP_FRACS]


@dataclass
class Inputs:
    q: torch.Tensor       # bf16 [B, H, N, d]
    k: torch.Tensor       # bf16 [B, H, N, d]
    v: torch.Tensor       # bf16 [B, H, N, d]
    proj_q: torch.Tensor  # fp32 [H, d, d]  (y = x @ W)
    proj_k: torch.Tensor  # fp32 [H, d, d]
    alpha: torch.Tensor   # fp32 [H, nq]
    topk_frac: float


def _block_offset(gen, B, H, N, d, std):
    off = torch.randn(B, H, N // BLOCK_K, d, generator=gen, dtype=torch.float32) * std
    return off.repeat_interleave(BLOCK_K, dim=2)


def make_inputs(w: Workload, heads: Optional[int] = None) -> Inputs:
    """Draw the workload's tensors on the CPU.

    ``heads`` limits the draw to the first ``heads`` heads: the draw order is
    per tensor, so a head subset is NOT a slice of the full draw. It is used for
    small reproducible cases; full-size parity draws every head.
    """
    H = w.H if heads is None else heads
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed)
    shape = (w.B, H, w.N, w.d)
    nq_ = torch.randn(shape, generator=gen, dtype=torch.float32)
    nk_ = torch.randn(shape, generator=gen, dtype=torch.float32)
    nv_ = torch.randn(shape, generator=gen, dtype=torch.float32)
    std = math.sqrt(w.offset_var)
    nq_ += _block_offset(gen, w.B, H, w.N, w.d, std)
    nk_ += _block_offset(gen, w.B, H, w.N, w.d, std)
    nv_ += _block_offset(gen, w.B, H, w.N, w.d, std)
    bias = torch.randn(w.B, H, 1, w.d, generator=gen, dtype=torch.float32)
    nk_ += bias
    pstd = 1.0 / math.sqrt(w.d)
    proj_q = torch.randn(H, w.d, w.d, generator=gen, dtype=torch.float32) * pstd
    proj_k = torch.randn(H, w.d, w.d, generator=gen, dtype=torch.float32) * pstd
    if w.alpha_one:
        alpha = torch.ones(H, w.nq, dtype=torch.float32)
    else:
        alpha = torch.rand(H, w.nq, generator=gen, dtype=torch.float32)
    return Inputs(
        q=nq_.to(torch.bfloat16),
        k=nk_.to(torch.bfloat16),
        v=nv_.to(torch.bfloat16),
        proj_q=proj_q.contiguous(),
        proj_k=proj_k.contiguous(),
        alpha=alpha.contiguous(),
        topk_frac=w.topk_frac,
    )


def make_custom(B, H, N, d, topk_frac, seed=0, offset_var=0.5, alpha_one=False) -> Inputs:
    """Inputs of an arbitrary shape drawn with the same recipe (edge-case tests)."""
    return make_inputs(Workload("custom", B, H, N, d, topk_frac, offset_var, seed, alpha_one))
