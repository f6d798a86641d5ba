"""Host logic of the multi-GPU ring on the CPU: the layout segments against the oracle's
position maps, the visiting schedule, the causal skip rule, and the real K||V exchange code
running on two and three gloo ranks with CPU tensors (after s steps, rank r holds the block
of position (r - s) mod W)."""

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import ring as A
from sequence_softmax_b200 import ring_dist


@pytest.mark.parametrize("layout,N,P", [("contiguous", 64, 4), ("striped", 60, 5), ("zigzag", 48, 3)])
def test_segments_match_oracle_positions(layout, N, P):
    want = A.layout_positions(layout, N, P)
    for p in range(P):
        toks = np.concatenate([t0 + st * np.arange(n) for t0, st, n in ring_dist.position_segments(layout, N, P, p)])
        assert np.array_equal(toks, want[p])


def test_schedule_visits_every_position_once():
    for W in (1, 2, 5, 8):
        for r in range(W):
            sched = ring_dist.ring_schedule(r, W)
            assert sched[0] == r and sorted(sched) == list(range(W))
            assert all(sched[s] == (r - s) % W for s in range(W))


def test_future_rule_matches_oracle_classes():
    N, P = 64, 4
    for layout in ("contiguous", "striped", "zigzag"):
        for a in range(P):
            for b in range(P):
                for qs in ring_dist.position_segments(layout, N, P, a):
                    for ks in ring_dist.position_segments(layout, N, P, b):
                        tq = qs[0] + qs[1] * np.arange(qs[2])
                        tk = ks[0] + ks[1] * np.arange(ks[2])
                        assert ring_dist.segment_in_future(qs, ks) == (A.chunk_class(tq, tk) == "skip")


def _rotate_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        buf = torch.full((2, 3), float(rank))
        nxt = torch.empty_like(buf)
        ex = ring_dist._Exchanger(None, buf)
        held = [int(buf[0, 0])]
        for _ in range(world - 1):
            h = ex.start(buf, nxt)
            nxt = ex.finish(h)
            buf, nxt = nxt, buf
            held.append(int(buf[0, 0]))
        out[rank] = held
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_rotates_blocks(world):
    out = mp.get_context("spawn").Manager().dict()
    port = 29600 + world + os.getpid() % 500
    mp.spawn(_rotate_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == ring_dist.ring_schedule(r, world)


class _OracleKernels:
    """Stand-ins for the library's backward kernels on CPU tensors (fp64 oracle), so that the
    ring's plumbing -- block rotation, accumulator hand-off and the return hop -- runs on gloo
    ranks without a GPU."""

    @staticmethod
    def backward_delta(o, d_o):
        import oracle
        return torch.from_numpy(oracle.delta(o.numpy(), d_o.numpy())).float()

    @staticmethod
    def partial_backward(q, k, v, d_o, lse, delta, dq_acc, dk_acc, dv_acc, causal=False, scale=None, q_tok0=0,
                         q_tok_stride=1, k_tok0=0, k_tok_stride=1):
        import oracle
        g = oracle.partial_backward(q.numpy(), k.numpy(), v.numpy(), d_o.numpy(), lse.numpy(), delta.numpy(), scale,
                                    causal, q_tok0, q_tok_stride, k_tok0, k_tok_stride)
        for acc, x in zip((dq_acc, dk_acc, dv_acc), g):
            acc += torch.from_numpy(x).float()


def _bwd_main(rank, world, port, layout, causal, out):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 1, 2, 24 * world, 8
        r = np.random.default_rng(5)
        q, k, v, do = (r.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(4))
        o, lse = oracle.attention(q, k, v, d ** -0.5, causal)
        idx = np.concatenate([t0 + st * np.arange(n) for t0, st, n in ring_dist.position_segments(layout, N, world, rank)])
        loc = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, :, idx])).float()  # noqa: E731
        g = ring_dist.ring_backward_dist(loc(q), loc(k), loc(v), loc(o), loc(do), loc(lse), N, layout, causal,
                                         kernels=_OracleKernels)
        out[rank] = (idx, [t.numpy() for t in g])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal", [(2, "contiguous", True), (3, "zigzag", True), (2, "striped", True),
                                                 (3, "contiguous", False)])
def test_ring_backward_plumbing(world, layout, causal):
    """ring_backward_dist on gloo ranks gives the definition's gradients for every rank's tokens."""
    import oracle
    out = mp.get_context("spawn").Manager().dict()
    port = 29650 + 7 * world + os.getpid() % 400
    mp.spawn(_bwd_main, args=(world, port, layout, causal, out), nprocs=world, join=True)
    B, H, N, d = 1, 2, 24 * world, 8
    r = np.random.default_rng(5)
    q, k, v, do = (r.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(4))
    ref = oracle.attention_backward(q, k, v, do, d ** -0.5, causal)
    for rk in range(world):
        idx, got = out[rk]
        for gg, rr in zip(got, ref):
            assert np.abs(gg - rr[:, :, idx]).max() <= 1e-4 * max(1.0, np.abs(rr).max())
