"""Host logic of the peer-memory ring (``peer_ring``) on the CPU: gloo ranks whose "peer
memory" is shared-memory CPU tensors, with the library's kernels replaced by the fp64
oracle. The ring reads every block from its owner's buffer and, in the backward, adds each
block's dK and dV into its owner's accumulators in place, one writer per block per step."""

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sequence_softmax_b200 import peer_ring, ring_dist

from .test_ring_dist_host import _OracleKernels


class _OracleForwardKernels:
    """Stand-ins for ``partial_fold`` (with ``partial`` and ``merge``) on CPU tensors (fp64 oracle)."""

    @staticmethod
    def partial_fold(q, k, v, o_state, lse_state, causal=False, scale=None, q_tok0=0, q_tok_stride=1, k_tok0=0,
                     k_tok_stride=1, k_norm_max=None):
        import oracle
        o, l = oracle.partial(q.numpy(), k.numpy(), v.numpy(), scale, causal, q_tok0, q_tok_stride, k_tok0,
                              k_tok_stride)
        mo, ml = oracle.merge(np.stack([o_state.numpy(), o]), np.stack([lse_state.numpy(), l]))
        o_state.copy_(torch.from_numpy(mo))
        lse_state.copy_(torch.from_numpy(ml))
        return o_state, lse_state

    @staticmethod
    def partial(q, k, v, causal=False, scale=None, q_tok0=0, q_tok_stride=1, k_tok0=0, k_tok_stride=1, out=None,
                lse=None):
        import oracle
        o, l = oracle.partial(q.numpy(), k.numpy(), v.numpy(), scale, causal, q_tok0, q_tok_stride, k_tok0,
                              k_tok_stride)
        out.copy_(torch.from_numpy(o))
        lse.copy_(torch.from_numpy(l))

    @staticmethod
    def merge(o_parts, lse_parts, out_dtype=torch.float32):
        import oracle
        o, l = oracle.merge(o_parts.numpy(), lse_parts.numpy())
        return torch.from_numpy(o).to(out_dtype), torch.from_numpy(l).float()


class _SharedPool:
    """Peer memory on the CPU: call i of ``share`` on rank r uses pool[i][r], a tensor in
    shared memory that every rank's process sees."""

    def __init__(self, pool):
        self.pool = pool
        self.calls = 0

    def __call__(self, local, group):
        slots = self.pool[self.calls]
        self.calls += 1
        rank = dist.get_rank(group)
        assert slots[rank].shape == local.shape and slots[rank].dtype == local.dtype
        slots[rank].copy_(local)

        class _Views:
            views = list(slots)

            @staticmethod
            def close():
                pass

        return _Views()


def _shapes(world, layout, N, B, H, d):
    nseg = len(ring_dist.position_segments(layout, N, world, 0))
    return (2, nseg, B, H, N // world // nseg, d)


def _inputs(world, causal):
    import oracle
    B, H, N, d = 1, 2, 24 * world, 8
    r = np.random.default_rng(5)
    q, k, v, do = (r.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(4))
    o, lse = oracle.attention(q, k, v, d ** -0.5, causal)
    return (B, H, N, d), q, k, v, do, o, lse


def _main(rank, world, port, layout, causal, pool, out, mode="direct"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        (B, H, N, d), q, k, v, do, o, lse = _inputs(world, causal)
        idx = np.concatenate([t0 + st * np.arange(n) for t0, st, n in ring_dist.position_segments(layout, N, world, rank)])
        loc = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, :, idx])).float()  # noqa: E731
        share = _SharedPool(pool)
        of, lf = peer_ring.ring_forward_peer(loc(q), loc(k), loc(v), N, layout, causal, kernels=_OracleForwardKernels,
                                             share=share, mode=mode)
        g = peer_ring.ring_backward_peer(loc(q), loc(k), loc(v), loc(o), loc(do), loc(lse), N, layout, causal,
                                         kernels=_OracleKernels, share=share, mode=mode)
        out[rank] = (idx, of.numpy(), lf.numpy(), [t.numpy() for t in g])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal,mode", [(2, "contiguous", True, "direct"), (3, "zigzag", True, "direct"),
                                                      (2, "striped", True, "direct"), (3, "contiguous", False, "direct"),
                                                      (3, "zigzag", True, "copy"), (2, "striped", True, "copy"),
                                                      (4, "contiguous", False, "copy")])
def test_peer_ring_forward_and_backward(world, layout, causal, mode):
    """Every rank's O, lse, dQ, dK and dV equal the definition's for its tokens."""
    import oracle
    (B, H, N, d), q, k, v, do, o, lse = _inputs(world, causal)
    shp = _shapes(world, layout, N, B, H, d)
    # share calls in order: forward K||V, backward K||V, backward dK||dV accumulators
    pool = [[torch.zeros(shp).share_memory_() for _ in range(world)] for _ in range(3)]
    out = mp.get_context("spawn").Manager().dict()
    port = 29550 + 5 * world + (2 if mode == "copy" else 0) + os.getpid() % 400
    mp.spawn(_main, args=(world, port, layout, causal, pool, out, mode), nprocs=world, join=True)
    ref = oracle.attention_backward(q, k, v, do, d ** -0.5, causal)
    for rk in range(world):
        idx, of, lf, got = out[rk]
        assert np.abs(of - o[:, :, idx]).max() <= 1e-5
        assert np.abs(lf - lse[:, :, idx]).max() <= 1e-5
        for gg, rr in zip(got, ref):
            assert np.abs(gg - rr[:, :, idx]).max() <= 1e-4 * max(1.0, np.abs(rr).max())


def _order_main(rank, world, port, out):
    import random
    import time as _time

    from sequence_softmax_b200 import peer_ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rnd = random.Random(rank)
        spans = []
        for _call in range(2):  # two calls: the second must not see the first one's keys
            order = peer_ring._StepOrder(None, None)
            for s in range(world):
                order.before_step(s)
                t0 = _time.time()
                _time.sleep(rnd.uniform(0.0, 0.05))
                spans.append((_call, s, t0, _time.time()))
                order.after_step(s)
        out[rank] = spans
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_step_order_follows_the_predecessor(world):
    """Step s of rank r starts only after step s - 1 of rank r - 1 (the previous writer of
    the block rank r writes at step s) has ended, in every call."""
    out = mp.get_context("spawn").Manager().dict()
    port = 29750 + 13 * world + os.getpid() % 300
    mp.spawn(_order_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        prev = {(c, s): (t0, t1) for c, s, t0, t1 in out[(r - 1) % world]}
        for c, s, t0, _ in out[r]:
            if s > 0:
                assert t0 >= prev[(c, s - 1)][1]
