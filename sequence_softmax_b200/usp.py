"""USP: Ulysses head split inside a group of GPUs plus the ring across groups.

"Ring Attention 논문 분석" (youngju.dev), listing ``hybrid_ulysses_ring_attention``: the
devices form an R x U mesh. Inside an intra group (U devices, e.g. one NVSwitch domain) an
all-to-all turns the sequence split into a head split; across the inter groups (R) the
ring of ``ring_dist`` runs on each device's heads; a second all-to-all restores the
sequence split. The page leaves its ``all_to_all_reshape`` undefined; the reading here:

  * global rank g = r * U + u; device (r, u) holds the u-th of U equal contiguous pieces of
    virtual ring position r's tokens (position r of the contiguous, striped or zig-zag
    layout over R positions), all H heads: [B, H, N / (R U), d];
  * seq -> head: device u of the intra group receives every member's piece for heads
    [u H/U, (u+1) H/U), concatenated in member order, i.e. position r's tokens in order:
    [B, H/U, N/R, d] -- exactly what ``ring_forward_dist`` takes for position r;
  * head -> seq is the inverse.

Every arithmetic step runs in the library's kernels (through ``ring_dist``); this module
only moves tensors with the process groups' all-to-all. NCCL groups exchange CUDA tensors
directly; gloo groups go through host copies.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import peer_ring, ring_dist


def usp_groups(R: int, U: int):
    """Create the intra (same r, U members) and inter (same u, R members) groups of an R x U
    mesh of the default group's ranks; every rank must call this, in the same order.
    Returns (intra_group, inter_group) of the calling rank."""
    world = dist.get_world_size()
    if R * U != world:
        raise ValueError(f"R x U = {R} x {U} does not cover {world} ranks")
    rank = dist.get_rank()
    intra = inter = None
    for r in range(R):
        g = dist.new_group([r * U + u for u in range(U)])
        if rank // U == r:
            intra = g
    for u in range(U):
        g = dist.new_group([r * U + u for r in range(R)])
        if rank % U == u:
            inter = g
    return intra, inter


def device_tokens(layout: str, N: int, R: int, U: int, r: int, u: int):
    """Global token indices held by device (r, u), in the order it holds them."""
    import numpy as np
    toks = np.concatenate([t0 + st * np.arange(n) for t0, st, n in ring_dist.position_segments(layout, N, R, r)])
    if len(toks) % U:
        raise ValueError("a position's tokens must split evenly over the intra group")
    m = len(toks) // U
    return toks[u * m:(u + 1) * m]


def _all_to_all(x: torch.Tensor, group) -> torch.Tensor:
    """all_to_all_single along dim 0 (equal splits), through host memory for gloo."""
    if dist.get_backend(group) == "nccl" or not x.is_cuda:
        out = torch.empty_like(x)
        dist.all_to_all_single(out, x.contiguous(), group=group)
        return out
    xh = x.cpu()
    out = torch.empty_like(xh)
    dist.all_to_all_single(out, xh, group=group)
    return out.to(x.device)


def seq_to_head(x: torch.Tensor, group) -> torch.Tensor:
    """[B, H, S, ...] sequence piece of every member -> [B, H/U, U S, ...] head group of this member."""
    U = dist.get_world_size(group)
    B, H, S = x.shape[:3]
    rest = tuple(x.shape[3:])
    if H % U:
        raise ValueError("heads must split evenly over the intra group")
    parts = x.reshape(B, U, H // U, S, *rest).movedim(1, 0).contiguous()  # part u -> member u
    got = _all_to_all(parts, group)                                      # part u <- member u
    return got.movedim(0, 2).reshape(B, H // U, U * S, *rest)


def head_to_seq(y: torch.Tensor, group) -> torch.Tensor:
    """Inverse of seq_to_head: [B, H/U, U S, ...] -> [B, H, S, ...]."""
    U = dist.get_world_size(group)
    B, Hg, US = y.shape[:3]
    rest = tuple(y.shape[3:])
    S = US // U
    parts = y.reshape(B, Hg, U, S, *rest).movedim(2, 0).contiguous()  # part u = member u's tokens
    got = _all_to_all(parts, group)                                  # part u = head group u
    return got.movedim(0, 1).reshape(B, U * Hg, S, *rest)


def _ring_fns(ring: str):
    """The inter-group ring: "message" (``ring_dist``: K||V sent each step) or "peer"
    (``peer_ring``: K/V read in place from the owner's memory)."""
    if ring == "message":
        return ring_dist.ring_forward_dist, ring_dist.ring_backward_dist, {}
    if ring == "peer":
        return peer_ring.ring_forward_peer, peer_ring.ring_backward_peer, None
    raise ValueError(f"unknown ring {ring!r}")


def usp_forward(q, k, v, N: int, layout: str = "contiguous", causal: bool = False, scale: float | None = None,
                intra_group=None, inter_group=None, kernels=None, ring: str = "message", share=None):
    """Exact attention with the USP split. q, k, v: [B, H, N/(R U), d], this device's tokens
    (``device_tokens``). Returns (O [B, H, N/(R U), d], lse [B, H, N/(R U)] fp32).
    ``ring`` selects the inter-group ring ("message" or "peer"; ``share`` is passed to the
    peer ring)."""
    fwd, _, extra = _ring_fns(ring)
    extra = {"share": share} if extra is None else extra
    scale = q.shape[-1] ** -0.5 if scale is None else float(scale)
    qh, kh, vh = (seq_to_head(t, intra_group) for t in (q, k, v))
    o, lse = fwd(qh, kh, vh, N, layout, causal, scale, group=inter_group, kernels=kernels, **extra)
    return head_to_seq(o, intra_group), head_to_seq(lse, intra_group)


def usp_backward(q, k, v, o, d_o, lse, N: int, layout: str = "contiguous", causal: bool = False,
                 scale: float | None = None, intra_group=None, inter_group=None, kernels=None, ring: str = "message",
                 share=None):
    """Gradients (dQ, dK, dV) of ``usp_forward``'s output for upstream gradient d_o, all in this
    device's sequence piece [B, H, N/(R U), d]. ``ring`` and ``share`` as in ``usp_forward``."""
    _, bwd, extra = _ring_fns(ring)
    extra = {"share": share} if extra is None else extra
    scale = q.shape[-1] ** -0.5 if scale is None else float(scale)
    qh, kh, vh, oh, doh = (seq_to_head(t, intra_group) for t in (q, k, v, o, d_o))
    lh = seq_to_head(lse, intra_group)
    grads = bwd(qh, kh, vh, oh, doh, lh, N, layout, causal, scale, group=inter_group, kernels=kernels, **extra)
    return tuple(head_to_seq(g, intra_group) for g in grads)
