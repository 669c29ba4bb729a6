"""Seeded synthetic inputs for the MXFP8 GEMM workloads.

This module holds only random-number recipes (shapes, distributions, routing
structure).  It contains none of the quantisation or GEMM arithmetic, so the
CUDA path and the CPU oracle can both be fed from it without sharing any of
the method.

Workloads (the shapes are the ones the pages quote; the data is synthetic,
because the pages measure on DeepSeek-V3 training, whose data and weights are
not available here):
  * ``pr1``        128x256x512 dense; A ~ N(0,1), B ~ N(0,0.02).
  * ``page``       dense 64x2112x7168, 64x24576x1536, 128x7168x2048 (the
                   CUTLASS comparison table of the DeepGEMM summary page);
                   A ~ N(0,1) with 0.5% of entries x64, B ~ N(0,0.02).
  * ``large``      dense M=8192, (N,K) in {(7168,2048),(2112,7168),(4096,7168)};
                   row i of A = 2^u_i * N(0,1), u_i ~ U[-4,4]; B ~ N(0,0.02).
  * ``contiguous`` 32 experts, 8192 tokens x top-8 distinct experts drawn with
                   p(e) ~ (e+1)^-1.1 (Zipf, s=1.1); each expert's rows padded
                   to a multiple of 128 with zero rows; gate/up N=4096 K=7168,
                   down N=7168 K=2048 (fresh N(0,1) activations).
  * ``masked``     32 experts x 256 rows, masked_m[e] ~ U{0..256}; rows at or
                   beyond masked_m[e] are NaN; N=4096 K=7168.
  * ``moe_layer``  the ``contiguous`` routing as an explicit [8192, 8] table of
                   expert ids (same Zipf draw) with softmax gate weights over
                   N(0,1) logits; token activations [8192, 7168] ~ N(0,1).

All draws come from ``torch.Generator`` objects seeded explicitly; on a CUDA
device the CUDA generator is used (same recipe, different stream of numbers),
which keeps full-size generation fast.  Values are drawn in fp32 and rounded
to BF16 (round-to-nearest-even, torch's cast).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

PAGE_SHAPES = [(64, 2112, 7168), (64, 24576, 1536), (128, 7168, 2048)]
LARGE_NK = [(7168, 2048), (2112, 7168), (4096, 7168)]
LARGE_M = 8192

MOE_EXPERTS = 32
MOE_TOKENS = 8192
MOE_TOPK = 8
MOE_ZIPF_S = 1.1
MOE_GATE_NK = (4096, 7168)
MOE_DOWN_NK = (7168, 2048)

MASKED_EXPERTS = 32
MASKED_MAX_M = 256
MASKED_NK = (4096, 7168)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def outlier_bf16(shape, seed: int, frac: float = 0.005, scale: float = 64.0, device="cpu"):
    """N(0,1) with a Bernoulli(frac) subset of entries multiplied by ``scale``."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    hit = torch.rand(shape, generator=g, device=device) < frac
    x = torch.where(hit, x * scale, x)
    return x.to(torch.bfloat16)


def row_loguniform_bf16(shape, seed: int, lo: float = -4.0, hi: float = 4.0, device="cpu"):
    """Row i is 2^u_i * N(0,1) with u_i ~ U[lo, hi]."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    u = torch.rand(shape[:-1] + (1,), generator=g, device=device) * (hi - lo) + lo
    return (x * torch.exp2(u)).to(torch.bfloat16)


# ---------------------------------------------------------------- dense

def dense_problem(m: int, n: int, k: int, seed: int = 0, kind: str = "normal", device="cpu"):
    """(A [m,k], B [n,k]) BF16 for one dense GEMM D = A B^T."""
    if kind == "normal":
        a = normal_bf16((m, k), 1.0, seed, device)
    elif kind == "outlier":
        a = outlier_bf16((m, k), seed, device=device)
    elif kind == "loguniform":
        a = row_loguniform_bf16((m, k), seed, device=device)
    else:
        raise ValueError(kind)
    b = normal_bf16((n, k), 0.02, seed + 1_000_003, device)
    return a, b


# ---------------------------------------------------------------- MoE routing

def zipf_routing_counts(tokens: int = MOE_TOKENS, experts: int = MOE_EXPERTS, topk: int = MOE_TOPK,
                        s: float = MOE_ZIPF_S, seed: int = 0) -> torch.Tensor:
    """Rows per expert when each token picks ``topk`` distinct experts, drawn
    without replacement with p(e) proportional to (e+1)^-s."""
    g = _gen(seed, "cpu")
    p = torch.arange(1, experts + 1, dtype=torch.float64).pow(-s)
    p = (p / p.sum()).expand(tokens, experts).contiguous()
    choice = torch.multinomial(p, topk, replacement=False, generator=g)
    return torch.bincount(choice.flatten(), minlength=experts).to(torch.int64)


def topk_ids(tokens: int = MOE_TOKENS, topk: int = MOE_TOPK, experts: int = MOE_EXPERTS, seed: int = 0,
             s: float = MOE_ZIPF_S):
    """Routing table int32 numpy [tokens, topk]: each token's ``topk``
    distinct experts, drawn without replacement with p(e) proportional to
    (e+1)^-s (the router's choice; the router itself is not modelled)."""
    g = _gen(seed, "cpu")
    p = torch.arange(1, experts + 1, dtype=torch.float64).pow(-s)
    p = (p / p.sum()).expand(tokens, experts).contiguous()
    choice = torch.multinomial(p, topk, replacement=False, generator=g)
    return choice.to(torch.int32).numpy()


def gate_weights(tokens: int = MOE_TOKENS, topk: int = MOE_TOPK, seed: int = 0):
    """Gate weights float32 numpy [tokens, topk]: a softmax over N(0,1)
    logits per token (positive, summing to 1 like a top-k router's)."""
    g = _gen(seed + 17, "cpu")
    logits = torch.randn(tokens, topk, generator=g, dtype=torch.float32)
    return torch.softmax(logits, dim=1).numpy()


def padded_offsets(counts: torch.Tensor, align: int = 128) -> torch.Tensor:
    """int32 [E+1] start rows of each expert with every group padded to ``align``."""
    padded = (counts + align - 1) // align * align
    off = torch.zeros(len(counts) + 1, dtype=torch.int64)
    off[1:] = torch.cumsum(padded, 0)
    return off.to(torch.int32)


@dataclass
class ContiguousProblem:
    counts: torch.Tensor            # int64 [E]  real rows per expert
    offsets: torch.Tensor           # int32 [E+1] padded group starts
    a: torch.Tensor                 # bf16 [M_total, K]  (padding rows are zero)
    b: torch.Tensor                 # bf16 [E, N, K]
    real_rows: int = field(default=0)


def contiguous_problem(n: int, k: int, seed: int = 0, counts: torch.Tensor | None = None,
                       experts: int = MOE_EXPERTS, device="cpu", act_seed: int | None = None):
    """A_cat with each expert's real rows followed by zero padding rows."""
    if counts is None:
        counts = zipf_routing_counts(experts=experts, seed=seed)
    off = padded_offsets(counts)
    m_total = int(off[-1])
    a = normal_bf16((m_total, k), 1.0, seed + 7 if act_seed is None else act_seed, device)
    row = torch.arange(m_total, device=device)
    valid = torch.zeros(m_total, dtype=torch.bool, device=device)
    for e in range(len(counts)):
        s0 = int(off[e])
        valid |= (row >= s0) & (row < s0 + int(counts[e]))
    a = torch.where(valid[:, None], a, torch.zeros((), dtype=a.dtype, device=device))
    b = normal_bf16((len(counts), n, k), 0.02, seed + 2_000_003, device)
    return ContiguousProblem(counts=counts, offsets=off, a=a, b=b, real_rows=int(counts.sum()))


@dataclass
class MaskedProblem:
    masked_m: torch.Tensor          # int32 [E]
    a: torch.Tensor                 # bf16 [E, max_m, K]; rows >= masked_m[e] are NaN
    b: torch.Tensor                 # bf16 [E, N, K]


def masked_counts(experts: int = MASKED_EXPERTS, max_m: int = MASKED_MAX_M, seed: int = 0):
    g = _gen(seed + 11, "cpu")
    return torch.randint(0, max_m + 1, (experts,), generator=g, dtype=torch.int64).to(torch.int32)


def masked_problem(n: int = MASKED_NK[0], k: int = MASKED_NK[1], experts: int = MASKED_EXPERTS,
                   max_m: int = MASKED_MAX_M, seed: int = 0, masked_m: torch.Tensor | None = None,
                   device="cpu"):
    if masked_m is None:
        masked_m = masked_counts(experts, max_m, seed)
    a = normal_bf16((experts, max_m, k), 1.0, seed + 13, device)
    row = torch.arange(max_m, device=device)[None, :]
    pad = row >= masked_m.to(device)[:, None].to(torch.int64)
    a = torch.where(pad[:, :, None], torch.full((), float("nan"), dtype=a.dtype, device=device), a)
    b = normal_bf16((experts, n, k), 0.02, seed + 3_000_017, device)
    return MaskedProblem(masked_m=masked_m, a=a, b=b)
