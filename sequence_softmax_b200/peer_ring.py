"""Ring attention across GPUs with every K/V block read from its owner's memory
(``ring_forward_peer``, ``ring_backward_peer``).

``ring_dist`` moves K||V to the successor at every step with the process group's
point-to-point calls. GPUs joined by NVLink / NVSwitch can address each other's memory, so
here no message is sent: each rank maps the other ranks' K||V buffers once (CUDA IPC
handles, exchanged through the process group) and at step s reads block (rank - s) mod W
from its owner. Visiting order, causal skip and the online-softmax merge are those of
``ring_dist`` ("Ring Attention 논문 분석", listing ``ring_attention_forward``; gpumode
lecture 013 notes, log-sum-exp merge), with the same kernels on the same values in the same
order, so the two give bit-identical results.

How K||V is read (``mode``): "copy" (the default) pulls each step's block one step ahead
into a local double buffer with one DMA copy (``cudaMemcpyAsync`` on a copy stream), so the
block crosses NVLink once while the previous step computes, and the kernels' re-reads of
its tiles (every query tile pair streams the whole block) stay in this GPU's L2 and memory:
the "receive into local memory, then local TMA" plan. "direct" hands the kernels the
owner's pointers, so their TMA loads fetch every tile over NVLink as the MMA pipeline
consumes it, re-reads included.

Backward: block c's fp32 dK and dV accumulators live in c's owner's memory. At step s the
rank holding block (rank - s) mod W adds its queries' contributions into them in place
(``ra_partial_backward`` stores through the mapped pointers) and into its own dQ. Block c
is written by rank c + s at step s; each writer's stream waits, through an interprocess
CUDA event, for the previous writer's kernels (``_StepOrder``), so there is one writer per
block at a time without any host waiting for GPU work, and when the last step ends each
owner holds its blocks' dK and dV: the listing ``ring_attention_backward``'s reduce, read
as that sum, with no return hop.

Only the library's kernels and the DMA copies touch another rank's memory (plain per-CTA
TMA loads, the backward's accumulator stores, ``cudaMemcpyAsync``); merges, casts
and other copies run on local buffers.
Buffers are shared through ``share(tensor, group)`` (default: ``PeerBuffers``), which
returns an object whose ``views[r]`` is rank r's buffer and whose ``close()`` unmaps them.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding
from .ring_dist import _split_segments, position_segments, ring_schedule, segment_in_future


def _cuda_api():
    try:
        from cuda.bindings import driver, runtime
    except ImportError as e:  # pragma: no cover - the image ships cuda-python
        raise RuntimeError("the peer-memory ring needs cuda-python (cuda.bindings) for CUDA IPC") from e
    return driver, runtime


def _ok(res, what: str):
    """cuda-python returns (status, outputs...): raise on a failed status, else the outputs."""
    if int(res[0]) != 0:
        raise RuntimeError(f"{what} failed: {res[0]}")
    out = res[1:]
    return out[0] if len(out) == 1 else out


class _DeviceArray:
    """A raw device pointer in the CUDA array interface, so torch can view it without a copy."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (int(ptr), False),
                                         "version": 3}


# torch dtype -> (array-interface type of the same width, torch dtype of that type)
_VIEW_TYPES = {torch.bfloat16: ("<i2", torch.int16), torch.float32: ("<f4", torch.float32)}

# Remote allocations mapped by this process: IPC handle bytes -> [device pointer, users].
# PyTorch's caching allocator can place several tensors in one allocation, whose handles
# are then identical; each allocation is mapped once and unmapped with its last user.
_MAPPED: dict = {}


def _map(runtime, raw: bytes) -> int:
    ent = _MAPPED.get(raw)
    if ent is None:
        h = runtime.cudaIpcMemHandle_t()
        h.reserved = raw
        ptr = _ok(runtime.cudaIpcOpenMemHandle(h, runtime.cudaIpcMemLazyEnablePeerAccess), "cudaIpcOpenMemHandle")
        ent = _MAPPED[raw] = [int(ptr), 0]
    ent[1] += 1
    return ent[0]


def _unmap(runtime, raw: bytes):
    ent = _MAPPED[raw]
    ent[1] -= 1
    if ent[1] == 0:
        del _MAPPED[raw]
        _ok(runtime.cudaIpcCloseMemHandle(ent[0]), "cudaIpcCloseMemHandle")


class PeerBuffers:
    """Every rank's buffer of one shape and dtype, mapped into this process.

    ``views[r]`` is rank r's buffer (``views[rank]`` is ``local`` itself); a remote view's
    torch device may name the owner's GPU, and only its pointer is meant to be used. The mapping uses
    legacy CUDA IPC: the handle covers the allocation that holds ``local``, and the offset of
    ``local`` inside it travels with the handle. ``close()`` unmaps the remote buffers; call
    it only when no launched kernel reads them any more.
    """

    def __init__(self, local: torch.Tensor, group=None):
        if not local.is_cuda or not local.is_contiguous() or local.dtype not in _VIEW_TYPES:
            raise ValueError("PeerBuffers needs a contiguous CUDA tensor of bf16 or fp32")
        self.rank = dist.get_rank(group)
        self._opened = []
        if dist.get_world_size(group) == 1:
            self.views = [local]
            return
        driver, runtime = _cuda_api()
        _ok(driver.cuInit(0), "cuInit")
        base, _size = _ok(driver.cuMemGetAddressRange(local.data_ptr()), "cuMemGetAddressRange")
        handle = _ok(runtime.cudaIpcGetMemHandle(int(base)), "cudaIpcGetMemHandle")
        mine = (bytes(handle.reserved), local.data_ptr() - int(base), tuple(local.shape), str(local.dtype))
        infos = [None] * dist.get_world_size(group)
        dist.all_gather_object(infos, mine, group=group)
        typestr, view_dtype = _VIEW_TYPES[local.dtype]
        self.views = []
        try:
            for r, (raw, offset, shape, dtype) in enumerate(infos):
                if r == self.rank:
                    self.views.append(local)
                    continue
                if shape != tuple(local.shape) or dtype != str(local.dtype):
                    raise ValueError("every rank must share a buffer of the same shape and dtype")
                rbase = _map(runtime, raw)
                self._opened.append(raw)
                # No device argument: torch takes the device from the pointer (possibly the
                # owner's GPU) and never copies. The view is only handed to the library and to
                # DMA copies as a pointer; no torch operation that launches a kernel touches it.
                t = torch.as_tensor(_DeviceArray(rbase + offset, shape, typestr))
                if t.data_ptr() != rbase + offset:
                    raise RuntimeError("a peer buffer view must alias the mapped memory")
                self.views.append(t if view_dtype == local.dtype else t.view(local.dtype))
        except Exception:
            self.close()
            raise

    def close(self):
        self.views = []
        opened, self._opened = self._opened, []
        if opened:
            _, runtime = _cuda_api()
            for raw in opened:
                _unmap(runtime, raw)


def _fence(group, device_work: bool):
    """Every rank's launched work is complete before any rank goes on."""
    if device_work:
        torch.cuda.current_stream().synchronize()
    dist.barrier(group)


# _StepOrder instances created so far per group (by its global ranks): every member makes
# them in the same order, so the count names an instance consistently across processes.
_ORDER_SEQ: dict = {}


class _StepOrder:
    """Device-side order between consecutive writers of a block's dK/dV accumulators.

    At step s rank r adds into the accumulators of block (r - s) mod W, which rank r - 1
    wrote at step s - 1. After enqueueing step s, every rank records its interprocess CUDA
    event for step s on its stream and publishes that in the process group's store; before
    step s + 1, its successor waits (on the host) for that key only, then makes its stream
    wait on the event (cudaStreamWaitEvent). No host waits for GPU work, so the steps'
    kernels queue back to back, and each event is recorded once per call, so a wait always
    refers to the intended step. Without CUDA (host tensors) the key alone orders the steps.
    """

    def __init__(self, group, device: torch.device | None):
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.cuda = device is not None
        if self.world == 1:
            return
        ranks = tuple(dist.get_process_group_ranks(group) if group is not None else range(self.world))
        seq = _ORDER_SEQ.get(ranks, 0)
        _ORDER_SEQ[ranks] = seq + 1
        self.prefix = f"ra_peer_ring_order/{'-'.join(map(str, ranks))}/{seq}"
        self.store = dist.distributed_c10d._get_default_store()
        if self.cuda:
            self.mine = [torch.cuda.Event(interprocess=True) for _ in range(self.world)]
            handles = [None] * self.world
            dist.all_gather_object(handles, [e.ipc_handle() for e in self.mine], group=group)
            prev = (self.rank - 1) % self.world
            self.pred = [torch.cuda.Event.from_ipc_handle(device, h) for h in handles[prev]]

    def after_step(self, s: int):
        """Step s's kernels are enqueued: publish their completion to the successor."""
        if self.world == 1:
            return
        if self.cuda:
            self.mine[s].record(torch.cuda.current_stream())
        self.store.set(f"{self.prefix}/{self.rank}/{s}", "1")

    def before_step(self, s: int):
        """Step s may write what the predecessor wrote at step s - 1: wait for it."""
        if s == 0 or self.world == 1:
            return
        self.store.wait([f"{self.prefix}/{(self.rank - 1) % self.world}/{s - 1}"])
        if self.cuda:
            torch.cuda.current_stream().wait_event(self.pred[s - 1])


class _Blocks:
    """The K||V block of each ring step, as the tensor this rank's kernels read.

    "direct": the owner's buffer itself; the kernels' TMA loads fetch every tile they read
    over NVLink, including the re-reads (each query tile pair streams the whole block).
    "copy": a local double buffer. While step s computes, the block of step s + 1 is pulled
    from its owner with one DMA copy (``cudaMemcpyAsync``) on a copy stream, so each block
    crosses NVLink once, the transfer overlaps the compute, and the re-reads hit this GPU's
    L2 and memory. Call ``get(s)`` and ``done(s)`` in step order.
    """

    def __init__(self, mode: str, peers, sched, local_kv: torch.Tensor):
        if mode not in ("direct", "copy"):
            raise ValueError(f"unknown mode {mode!r}")
        self.mode, self.peers, self.sched = mode, peers, sched
        self.cuda = local_kv.is_cuda
        if mode == "copy" and len(sched) > 1:
            self.bufs = [torch.empty_like(local_kv) for _ in range(2)]
            self.copy_stream = torch.cuda.Stream(device=local_kv.device) if self.cuda else None
            self.ready = [None, None]  # copy into bufs[i] complete
            self.freed = [None, None]  # the kernels that read bufs[i] complete

    def get(self, s: int) -> torch.Tensor:
        """Block of step s; in "copy" mode also starts the pull of step s + 1's block."""
        if self.mode == "direct":
            return self.peers.views[self.sched[s]]
        if s + 1 < len(self.sched):
            self._pull((s + 1) % 2, self.peers.views[self.sched[s + 1]])
        if s == 0:
            return self.peers.views[self.sched[0]]  # this rank's own block
        if self.cuda:
            torch.cuda.current_stream().wait_event(self.ready[s % 2])
        return self.bufs[s % 2]

    def done(self, s: int):
        """Step s's kernels are enqueued; the buffer they read may be refilled after them."""
        if self.mode == "copy" and s > 0 and self.cuda:
            ev = torch.cuda.Event()
            ev.record(torch.cuda.current_stream())
            self.freed[s % 2] = ev

    def _pull(self, i: int, src: torch.Tensor):
        dst = self.bufs[i]
        if not self.cuda:
            dst.copy_(src)
            return
        if self.freed[i] is not None:
            self.copy_stream.wait_event(self.freed[i])
        _, runtime = _cuda_api()
        _ok(runtime.cudaMemcpyAsync(dst.data_ptr(), src.data_ptr(), dst.numel() * dst.element_size(),
                                    runtime.cudaMemcpyKind.cudaMemcpyDeviceToDevice,
                                    runtime.cudaStream_t(self.copy_stream.cuda_stream)), "cudaMemcpyAsync")
        ev = torch.cuda.Event()
        ev.record(self.copy_stream)
        self.ready[i] = ev


def _check_local(q_local, others, segs):
    if sum(s[2] for s in segs) != q_local.shape[2] or any(t.shape != q_local.shape for t in others):
        raise ValueError("local tensors must hold the N/W tokens of this rank's position")


def ring_forward_peer(q_local, k_local, v_local, N: int, layout: str = "contiguous", causal: bool = False,
                      scale: float | None = None, group=None, kernels=None, share=None, mode: str = "copy"):
    """Exact attention over N tokens split across the ranks of `group`, reading each K/V
    block from its owner's memory.

    Arguments and result as ``ring_dist.ring_forward_dist``: q_local, k_local, v_local
    [B, H, N/W, d] on this rank's GPU hold the tokens of virtual position `rank` in
    increasing token order; returns (O_local in the input dtype, lse_local fp32).
    ``kernels`` (default: the library binding) provides ``partial_fold`` and, for bf16,
    ``key_norm_max`` (each K segment's largest key norm per head, read where the segment lives,
    which lets the folding kernel skip row maxima). ``mode``:
    "copy" (the default: each block pulled into a local buffer one step ahead, so it crosses
    NVLink once; see ``_Blocks``) or "direct" (the kernels read the owner's buffer).
    """
    kern = binding if kernels is None else kernels
    share = PeerBuffers if share is None else share
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, n_local, d = q_local.shape
    segs = position_segments(layout, N, world, rank)
    _check_local(q_local, (k_local, v_local), segs)
    nseg = len(segs)
    scale = d ** -0.5 if scale is None else float(scale)
    dev = q_local.device

    q_s = _split_segments(q_local, nseg)
    # segment-major, so that each block segment is a contiguous [B, H, L, d] the kernels read in place
    kv = torch.stack([torch.stack(_split_segments(k_local, nseg)), torch.stack(_split_segments(v_local, nseg))])
    # running state (O fp32, lse) per query segment
    state = [(torch.zeros(*q.shape, device=dev, dtype=torch.float32),
              torch.full(q.shape[:3], float("-inf"), device=dev, dtype=torch.float32)) for q in q_s]
    peers = share(kv, group)
    try:
        sched = ring_schedule(rank, world)
        blocks = _Blocks(mode, peers, sched, kv)
        _fence(group, kv.is_cuda)  # every rank's K||V is in place before anyone reads it
        for s, src in enumerate(sched):
            kv_src = blocks.get(s)
            for ki, kseg in enumerate(position_segments(layout, N, world, src)):
                kmax = None
                for qi, qseg in enumerate(segs):
                    if causal and segment_in_future(qseg, kseg):
                        continue
                    if kmax is None and kv_src.dtype == torch.bfloat16:
                        kmax = kern.key_norm_max(kv_src[0, ki])
                    st_o, st_l = state[qi]
                    kern.partial_fold(q_s[qi], kv_src[0, ki], kv_src[1, ki], st_o, st_l, causal=causal, scale=scale,
                                      q_tok0=qseg[0], q_tok_stride=qseg[1], k_tok0=kseg[0], k_tok_stride=kseg[1],
                                      k_norm_max=kmax)
            blocks.done(s)
        _fence(group, kv.is_cuda)  # no rank unmaps or frees a buffer another may still read
    finally:
        peers.close()
    out = torch.cat([o for o, _ in state], dim=2).to(q_local.dtype)
    lse = torch.cat([l for _, l in state], dim=2)
    return out, lse


def ring_backward_peer(q_local, k_local, v_local, o_local, do_local, lse_local, N: int, layout: str = "contiguous",
                       causal: bool = False, scale: float | None = None, group=None, kernels=None, share=None,
                       mode: str = "copy"):
    """Gradients (dQ, dK, dV) of ``ring_forward_peer``'s output for upstream gradient
    do_local, every block's dK and dV accumulated in place in its owner's memory.

    Arguments as ``ring_dist.ring_backward_dist`` (lse_local: the forward's final lse);
    ``kernels`` (default: the library binding) provides ``backward_delta`` and
    ``partial_backward``. ``mode`` chooses how K||V is read, as in ``ring_forward_peer``; the
    dK and dV accumulators are always added into in the owner's memory (each key tile's
    sums are stored once per step). Returns (dQ, dK, dV) [B, H, N/W, d] in the input dtype.
    """
    kern = binding if kernels is None else kernels
    share = PeerBuffers if share is None else share
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, n_local, d = q_local.shape
    segs = position_segments(layout, N, world, rank)
    _check_local(q_local, (k_local, v_local, o_local, do_local), segs)
    nseg = len(segs)
    scale = d ** -0.5 if scale is None else float(scale)
    dev = q_local.device

    delta = kern.backward_delta(o_local, do_local)
    q_s, do_s = _split_segments(q_local, nseg), _split_segments(do_local, nseg)
    lse_s, delta_s = _split_segments(lse_local, nseg), _split_segments(delta, nseg)
    dq_s = [torch.zeros(q.shape, device=dev, dtype=torch.float32) for q in q_s]
    kv = torch.stack([torch.stack(_split_segments(k_local, nseg)), torch.stack(_split_segments(v_local, nseg))])
    acc = torch.zeros(kv.shape, device=dev, dtype=torch.float32)  # this rank's blocks' dK, dV
    peers_kv = share(kv, group)
    try:
        peers_acc = share(acc, group)
    except Exception:
        peers_kv.close()
        raise
    try:
        sched = ring_schedule(rank, world)
        blocks = _Blocks(mode, peers_kv, sched, kv)
        order = _StepOrder(group, kv.device if kv.is_cuda else None)
        _fence(group, kv.is_cuda)
        for s, src in enumerate(sched):
            order.before_step(s)
            kv_src, acc_src = blocks.get(s), peers_acc.views[src]
            for ki, kseg in enumerate(position_segments(layout, N, world, src)):
                for qi, qseg in enumerate(segs):
                    if causal and segment_in_future(qseg, kseg):
                        continue
                    kern.partial_backward(q_s[qi], kv_src[0, ki], kv_src[1, ki], do_s[qi], lse_s[qi], delta_s[qi],
                                          dq_s[qi], acc_src[0, ki], acc_src[1, ki], causal=causal, scale=scale,
                                          q_tok0=qseg[0], q_tok_stride=qseg[1], k_tok0=kseg[0], k_tok_stride=kseg[1])
            blocks.done(s)
            # block src's next writer (rank + 1, next step) starts after these additions
            order.after_step(s)
        _fence(group, kv.is_cuda)  # every rank's additions are complete before the owners read them
        own = peers_acc.views[rank]
        dk = torch.cat(list(own[0]), dim=2).to(k_local.dtype)
        dv = torch.cat(list(own[1]), dim=2).to(v_local.dtype)
    finally:
        peers_acc.close()
        peers_kv.close()
    dq = torch.cat(dq_s, dim=2).to(q_local.dtype)
    return dq, dk, dv
