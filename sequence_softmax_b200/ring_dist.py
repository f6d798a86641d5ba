"""Ring attention across GPUs: one process per GPU, K and V rotating around the ring
(forward: ``ring_forward_dist``; backward: ``ring_backward_dist``).

Each rank holds the query, key and value tokens of one virtual ring position (the
contiguous, striped or zig-zag layout of ``include/ra.h``) and keeps its query block for the
whole computation. At step s it receives the K and V of position (rank - s) mod W from its
predecessor and forwards the block it holds to its successor ("Ring Attention 논문 분석",
listing ``ring_attention_forward``; "Ring Attention" glossary, "How Ring Attention works").
K and V travel as one message (lecture 013 notes: one large message instead of two small
ones), posted before the step's compute so that the transfer overlaps it.

Every arithmetic step runs in the library's kernels: ``ra_partial_fold`` computes the
partial state of the local queries against the block held (skipped when the block is wholly
in the queries' future) and folds it into the running (O, lse) state in the same kernel --
the lse associativity of the lecture 013 notes applied step by step. PyTorch provides memory,
streams and the process group.

The exchange uses the process group's point-to-point operations: with NCCL on CUDA tensors
directly; with gloo (which only sends host tensors) through pinned host staging buffers.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


def position_segments(layout: str, N: int, P: int, p: int):
    """Token segments (tok0, stride, count) of virtual position p, in increasing token order."""
    if layout == "contiguous":
        if N % P:
            raise ValueError("contiguous layout needs N divisible by P")
        return [(p * (N // P), 1, N // P)]
    if layout == "striped":
        if N % P:
            raise ValueError("striped layout needs N divisible by P")
        return [(p, P, N // P)]
    if layout == "zigzag":
        if N % (2 * P):
            raise ValueError("zig-zag layout needs N divisible by 2P")
        c = N // (2 * P)
        return [(p * c, 1, c), ((2 * P - 1 - p) * c, 1, c)]
    raise ValueError(f"unknown layout {layout!r}")


def segment_in_future(q_seg, k_seg) -> bool:
    """True when every key token of k_seg is after every query token of q_seg (causal skip)."""
    q0, qs, qn = q_seg
    k0, ks, kn = k_seg
    return kn == 0 or qn == 0 or k0 > q0 + qs * (qn - 1)


def ring_schedule(rank: int, world: int):
    """Positions whose K/V rank `rank` holds at steps 0..world-1: (rank - s) mod world."""
    return [(rank - s) % world for s in range(world)]


def _peers(rank: int, world: int):
    return (rank + 1) % world, (rank - 1) % world


class _Exchanger:
    """Sends one tensor to the successor and receives the predecessor's into a second one."""

    def __init__(self, group, like: torch.Tensor):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.send_to, self.recv_from = _peers(self.rank, self.world)
        self.nccl = dist.get_backend(group) == "nccl"
        if not self.nccl:
            self.host_send = torch.empty(like.shape, dtype=like.dtype, pin_memory=like.is_cuda)
            self.host_recv = torch.empty(like.shape, dtype=like.dtype, pin_memory=like.is_cuda)

    def _gsend(self):
        return dist.get_global_rank(self.group, self.send_to) if self.group is not None else self.send_to

    def _grecv(self):
        return dist.get_global_rank(self.group, self.recv_from) if self.group is not None else self.recv_from

    def start(self, send: torch.Tensor, recv: torch.Tensor):
        """Post the exchange; returns a handle for ``finish``."""
        if self.nccl:
            ops = [dist.P2POp(dist.isend, send, self._gsend(), self.group),
                   dist.P2POp(dist.irecv, recv, self._grecv(), self.group)]
            return dist.batch_isend_irecv(ops), recv
        self.host_send.copy_(send)
        # even ranks send first, odd ranks receive first: no cycle of blocking sends
        if self.rank % 2 == 0:
            reqs = [dist.isend(self.host_send, self._gsend(), self.group),
                    dist.irecv(self.host_recv, self._grecv(), self.group)]
        else:
            reqs = [dist.irecv(self.host_recv, self._grecv(), self.group),
                    dist.isend(self.host_send, self._gsend(), self.group)]
        return reqs, recv

    def finish(self, handle):
        reqs, recv = handle
        for r in reqs:
            r.wait()
        if not self.nccl:
            recv.copy_(self.host_recv)
        return recv


def ring_forward_dist(q_local, k_local, v_local, N: int, layout: str = "contiguous", causal: bool = False,
                      scale: float | None = None, group=None, kernels=None):
    """Exact attention over a sequence of N tokens split across the ranks of `group`.

    q_local, k_local, v_local: [B, H, N/W, d] CUDA tensors (bf16 with d in {64, 128}, or fp32)
    holding the tokens of virtual position `rank` in increasing token order (for zig-zag,
    chunk rank followed by chunk 2W-1-rank). Returns (O_local [B, H, N/W, d] in the input
    dtype, lse_local [B, H, N/W] fp32) for the same tokens. ``kernels`` (default: the library
    binding) provides ``partial_fold`` and, for bf16, ``key_norm_max``: each received block's
    largest key norm per head, which lets the folding kernel skip row maxima.
    """
    kern = binding if kernels is None else kernels
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, n_local, d = q_local.shape
    segs = position_segments(layout, N, world, rank)
    if sum(s[2] for s in segs) != n_local or k_local.shape != q_local.shape or v_local.shape != q_local.shape:
        raise ValueError("local tensors must hold the N/W tokens of this rank's position")
    scale = d ** -0.5 if scale is None else float(scale)

    # Running state (O fp32, lse) per query segment, folded into by every visited block.
    dev = q_local.device
    q_segs, offs = [], 0
    for seg in segs:
        q_segs.append((q_local[:, :, offs:offs + seg[2]].contiguous(), seg, offs))
        offs += seg[2]
    state = [(torch.zeros(B, H, seg[2], d, device=dev, dtype=torch.float32),
              torch.full((B, H, seg[2]), float("-inf"), device=dev, dtype=torch.float32)) for _, seg, _ in q_segs]

    kv = torch.stack([k_local, v_local]).contiguous()     # one K||V message
    kv_next = torch.empty_like(kv)
    ex = _Exchanger(group, kv) if world > 1 else None
    for s, src in enumerate(ring_schedule(rank, world)):
        handle = ex.start(kv, kv_next) if (ex is not None and s < world - 1) else None
        k_segs = position_segments(layout, N, world, src)
        koff = 0
        for kseg in k_segs:
            kk = kv[0][:, :, koff:koff + kseg[2]].contiguous() if len(k_segs) > 1 else kv[0]
            vv = kv[1][:, :, koff:koff + kseg[2]].contiguous() if len(k_segs) > 1 else kv[1]
            koff += kseg[2]
            kmax = None  # per segment, as the peer ring takes it: both rings fold identical values
            for (qs, qseg, _), (st_o, st_l) in zip(q_segs, state):
                if causal and segment_in_future(qseg, kseg):
                    continue
                if kmax is None and kk.dtype == torch.bfloat16:
                    kmax = kern.key_norm_max(kk)
                kern.partial_fold(qs, kk, vv, st_o, st_l, causal=causal, scale=scale, q_tok0=qseg[0],
                                  q_tok_stride=qseg[1], k_tok0=kseg[0], k_tok_stride=kseg[1], k_norm_max=kmax)
        if handle is not None:
            kv_next = ex.finish(handle)
            kv, kv_next = kv_next, kv

    out = torch.empty_like(q_local)
    lse = torch.empty(B, H, n_local, device=dev, dtype=torch.float32)
    for (qs, seg, off), (st_o, st_l) in zip(q_segs, state):
        out[:, :, off:off + seg[2]].copy_(st_o)
        lse[:, :, off:off + seg[2]].copy_(st_l)
    return out, lse


def _split_segments(t: torch.Tensor, nseg: int):
    """[B, H, nseg * L, ...] -> list of nseg contiguous [B, H, L, ...] blocks."""
    L = t.shape[2] // nseg
    return [t[:, :, s * L:(s + 1) * L].contiguous() for s in range(nseg)]


def ring_backward_dist(q_local, k_local, v_local, o_local, do_local, lse_local, N: int, layout: str = "contiguous",
                       causal: bool = False, scale: float | None = None, group=None, kernels=None):
    """Gradients (dQ, dK, dV) of ``ring_forward_dist``'s output for upstream gradient do_local.

    Every tensor holds this rank's position tokens as in ``ring_forward_dist``; lse_local is
    the forward's final lse for them. The ring of "Ring Attention 논문 분석" (youngju.dev),
    listing ``ring_attention_backward``, with its reduce read as a sum at the owner: each KV
    block travels with two fp32 accumulators for its dK and dV; at step s the rank holding
    block (rank - s) mod W adds its queries' contributions to them (``ra_partial_backward``,
    skipped when the block is wholly in the queries' future) and to its own dQ, then hands
    the accumulators on. After the last step one more hop brings every block's dK, dV back
    to its owner. K and V are sent ahead of the step's compute (the transfer overlaps it);
    the accumulators follow it. ``kernels`` (default: the library binding) provides
    ``backward_delta`` and ``partial_backward``.

    Returns (dQ, dK, dV) [B, H, N/W, d] in the input dtype.
    """
    kern = binding if kernels is None else kernels
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, n_local, d = q_local.shape
    segs = position_segments(layout, N, world, rank)
    nseg = len(segs)
    if sum(s[2] for s in segs) != n_local or any(t.shape != q_local.shape for t in (k_local, v_local, o_local,
                                                                                      do_local)):
        raise ValueError("local tensors must hold the N/W tokens of this rank's position")
    scale = d ** -0.5 if scale is None else float(scale)
    dev = q_local.device

    delta = kern.backward_delta(o_local, do_local)
    q_s, do_s = _split_segments(q_local, nseg), _split_segments(do_local, nseg)
    lse_s, delta_s = _split_segments(lse_local, nseg), _split_segments(delta, nseg)
    dq_s = [torch.zeros(q.shape, device=dev, dtype=torch.float32) for q in q_s]

    # Travelling block, segment-major so that every segment is a contiguous [B, H, L, d].
    kv = torch.stack([torch.stack(_split_segments(k_local, nseg)), torch.stack(_split_segments(v_local, nseg))])
    acc = torch.zeros(kv.shape, device=dev, dtype=torch.float32)  # dK, dV of the block held
    kv_next, acc_next = torch.empty_like(kv), torch.empty_like(acc)
    ex_kv = _Exchanger(group, kv) if world > 1 else None
    ex_acc = _Exchanger(group, acc) if world > 1 else None
    for s, src in enumerate(ring_schedule(rank, world)):
        handle = ex_kv.start(kv, kv_next) if (ex_kv is not None and s < world - 1) else None
        for ki, kseg in enumerate(position_segments(layout, N, world, src)):
            for qi, qseg in enumerate(segs):
                if causal and segment_in_future(qseg, kseg):
                    continue
                kern.partial_backward(q_s[qi], kv[0, ki], kv[1, ki], do_s[qi], lse_s[qi], delta_s[qi], dq_s[qi],
                                      acc[0, ki], acc[1, ki], causal=causal, scale=scale, q_tok0=qseg[0],
                                      q_tok_stride=qseg[1], k_tok0=kseg[0], k_tok_stride=kseg[1])
        if ex_acc is not None:
            # the block's accumulators move on with it; after the last step this hop returns
            # them to the block's owner
            acc_next = ex_acc.finish(ex_acc.start(acc, acc_next))
            acc, acc_next = acc_next, acc
        if handle is not None:
            kv_next = ex_kv.finish(handle)
            kv, kv_next = kv_next, kv

    dq = torch.cat(dq_s, dim=2).to(q_local.dtype)
    dk = torch.cat(list(acc[0]), dim=2).to(k_local.dtype)
    dv = torch.cat(list(acc[1]), dim=2).to(v_local.dtype)
    return dq, dk, dv
