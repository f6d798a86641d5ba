"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws random tensors and names
shapes. Both the CUDA path's tests/bench and the CPU oracle's tests take their inputs
from here, so the two sides see bit-identical Q, K and V.

Recipe:

* The 4-device toy of the "Ring Attention" glossary (section "How Ring Attention
  works"): a torch CPU generator seeded with 0, ``randn(3, 32, 16)`` split into q, k, v,
  fp32, viewed as [1, 1, 32, 16].
* Every other workload: a ``torch.Generator`` on the target device seeded with the
  workload's seed, ``randn`` in fp32 drawn in the order q, k, v, each of shape
  [B, H, N, d], i.i.d. N(0, 1), then cast to the workload dtype. A query scale (the
  "Q x 4" running-max stress case) is applied after the cast; scaling by a power of two
  is exact in bf16.
* Score ramp (``ramp_qkv``): every query is 4u plus small noise and every key of 128-key
  block b is (b x gamma) u plus a random component orthogonal to u (8 N(0, 1) per
  coordinate, projected), for one random unit vector u; V is N(0, 1).
  A query's largest score then grows by about ``jump_log2`` (in log2 units, at the default
  scale d^-1/2) from each key block to the next, so an online softmax that visits the
  blocks in token order sees its running maximum move at every block. ``spread`` (8 by
  default) scales the orthogonal component; with a small one the keys are nearly parallel
  to u and |q| max|k| is close to the largest score, so a norm bound on the scores is tight.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, masking, ring layout and input seed."""

    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str            # "f32" or "bf16"
    causal: bool
    n_chunks: int         # virtual ring positions P
    layout: str           # "contiguous" | "striped" | "zigzag"
    seed: int
    q_scale: float = 1.0
    emit_lse: bool = True
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return self.d ** -0.5

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def visible_pairs(self) -> int:
        """Visible (query, key) pairs per head: N^2, or N(N+1)/2 when causal."""
        return self.N * (self.N + 1) // 2 if self.causal else self.N * self.N

    def flops(self) -> int:
        """Algorithmic FLOPs of one forward: 2 GEMMs x 2 flops x d per visible pair."""
        return 4 * self.d * self.B * self.H * self.visible_pairs()


# The workloads the pages' ring is exercised on (shapes of the pages' long-context
# training sequences; i.i.d. normal values).
WORKLOADS = {
    w.name: w
    for w in [
        Workload("toy-4dev-seq32-d16", 1, 1, 32, 16, "f32", False, 4, "contiguous", 0,
                 notes="the glossary's 4-device simulation; output vs full softmax attention"),
        Workload("seq4k-d64-noncausal-8chunks", 2, 8, 4096, 64, "bf16", False, 8, "contiguous", 2),
        Workload("seq4k-d64-noncausal-8chunks-qx4", 2, 8, 4096, 64, "bf16", False, 8, "contiguous", 2,
                 q_scale=4.0, notes="Q scaled by 4 to stress the running-max rescale"),
        Workload("seq32k-d128-causal-contig8", 1, 32, 32768, 128, "bf16", True, 8, "contiguous", 3),
        Workload("seq128k-d128-causal-zigzag16", 1, 32, 131072, 128, "bf16", True, 16, "zigzag", 4),
        Workload("seq128k-d128-causal-striped16", 1, 32, 131072, 128, "bf16", True, 16, "striped", 4),
        Workload("seq1m-d128-causal-zigzag16", 1, 8, 1048576, 128, "bf16", True, 16, "zigzag", 5,
                 notes="1M-token causal zig-zag forward emitting O and per-row lse"),
        # Head subsets of the two benchmark workloads for profiler counter captures (about
        # 1 GB on the device): the kernels walk the heads one after another (head-major CTA
        # order), so per-head traffic and time match the full workloads'.
        Workload("seq1m-d128-causal-zigzag16-h1", 1, 1, 1048576, 128, "bf16", True, 16, "zigzag", 5,
                 notes="one head of the 1M-token workload (counter captures)"),
        Workload("seq128k-d128-causal-zigzag16-h4", 1, 4, 131072, 128, "bf16", True, 16, "zigzag", 4,
                 notes="four heads of the 128K-token zig-zag workload (backward counter captures)"),
    ]
}

BENCH_WORKLOAD = "seq1m-d128-causal-zigzag16"


def toy_qkv():
    """The glossary toy's inputs: seed 0, randn(3, 32, 16) -> q, k, v as [1, 1, 32, 16] fp32 (CPU)."""
    g = torch.Generator().manual_seed(0)
    q, k, v = torch.randn(3, 32, 16, generator=g)
    return q.view(1, 1, 32, 16), k.view(1, 1, 32, 16), v.view(1, 1, 32, 16)


def make_qkv(B: int, H: int, N: int, d: int, dtype=torch.bfloat16, seed: int = 0,
             device="cpu", q_scale: float = 1.0, Nk: int | None = None):
    """Seeded i.i.d. N(0,1) q [B,H,N,d], k/v [B,H,Nk,d] (Nk defaults to N), cast to dtype."""
    Nk = N if Nk is None else Nk
    g = torch.Generator(device=device).manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g, device=device, dtype=torch.float32).to(dtype)
    k = torch.randn(B, H, Nk, d, generator=g, device=device, dtype=torch.float32).to(dtype)
    v = torch.randn(B, H, Nk, d, generator=g, device=device, dtype=torch.float32).to(dtype)
    if q_scale != 1.0:
        q = q * q_scale
    return q, k, v


def workload_qkv(w: Workload, device="cpu", batch_offset: int = 0):
    """Inputs of a named workload. ``batch_offset`` shifts the seed (used for per-rank replicas)."""
    if w.name == "toy-4dev-seq32-d16":
        q, k, v = toy_qkv()
        return q.to(device), k.to(device), v.to(device)
    return make_qkv(w.B, w.H, w.N, w.d, w.torch_dtype, w.seed + 1000 * batch_offset, device, w.q_scale)


def sample_rows(N: int, n_chunks: int, layout: str, count: int = 4096, seed: int = 1234):
    """Query rows checked on long workloads: ``count`` seeded random rows plus rows 0, N-1
    and the first and last row of every chunk boundary of the layout's token chunks."""
    g = torch.Generator().manual_seed(seed)
    rnd = torch.randint(0, N, (count,), generator=g)
    parts = 2 * n_chunks if layout == "zigzag" else n_chunks
    c = N // parts
    edges = [0, N - 1]
    for i in range(1, parts):
        edges += [i * c - 1, i * c]
    rows = torch.unique(torch.cat([rnd, torch.tensor(edges)]))
    return rows.numpy()


RAMP_BLOCK = 128  # keys per block of the score ramp


def ramp_qkv(N: int, d: int, jump_log2: float, seed: int = 0, dtype=torch.bfloat16, device="cpu",
             B: int = 1, H: int = 1, block: int = RAMP_BLOCK, spread: float = 8.0):
    """Seeded q, k, v [B, H, N, d] whose scores rise by ~jump_log2 per `block`-key block
    (128 by default; 64 puts a jump in the middle of every 128-key tile as well).

    q_i = 4 u + 0.02 n_i, k_j = (floor(j / block) gamma) u + spread (I - u u^T) n'_j with gamma
    chosen so that 4 gamma d^-1/2 log2(e) = jump_log2; u is a unit vector, n, n' i.i.d.
    N(0, 1). The orthogonal part barely moves the scores (the queries are nearly parallel to
    u) but keeps the keys of one block apart: without it every key of the dominant block is
    the same vector, the rows of dS (which sum to zero) multiply it, and dQ is a small
    difference of large terms.
    """
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(d, generator=g, dtype=torch.float64)
    u /= u.norm()
    a = 4.0
    gamma = jump_log2 / (a * d ** -0.5 * 1.4426950408889634)
    blk = (torch.arange(N, dtype=torch.float64) // block)[:, None]
    q = a * u + 0.02 * torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    w = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    k = gamma * blk * u + spread * (w - (w @ u)[..., None] * u)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    return tuple(t.to(dtype).to(device) for t in (q, k, v))
