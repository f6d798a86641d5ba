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
