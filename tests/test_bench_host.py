"""Host-side logic of bench.py on the CPU: the max-over-ranks timing with two gloo ranks,
per-rank replica inputs, and the reference arm (the fp64 oracle timed on host cores)."""

import json
import os
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sequence_softmax_b200.inputs import WORKLOADS, workload_qkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    port = 29500 + os.getpid() % 1000
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1] == 15.0


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1, None) == 3.25


def test_rank_replicas_differ_but_share_shape():
    w = WORKLOADS["seq4k-d64-noncausal-8chunks"]
    small = type(w)(w.name + "-tiny", 1, 2, 64, 64, "bf16", False, 2, "contiguous", w.seed)
    a = workload_qkv(small, device="cpu", batch_offset=0)
    b = workload_qkv(small, device="cpu", batch_offset=1)
    assert a[0].shape == b[0].shape and not torch.equal(a[0], b[0])


def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "seq4k-d64-noncausal-8chunks", "--steps", "1", "--warmup", "0",
                        "--cpu-seconds", "1"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""


def _ring_main(rank, world, port, layout, causal, out):
    """The bench's ring mode on gloo ranks: each rank takes its position's tokens with
    bench.position_tokens and runs ring_dist.ring_forward_dist through bench.CountingKernels
    around oracle stand-ins for ra_partial / ra_merge."""
    import numpy as np

    from sequence_softmax_b200.ring_dist import position_segments, ring_forward_dist

    from .test_peer_ring_host import _OracleForwardKernels
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 1, 2, 16 * world, 8
        g = torch.Generator().manual_seed(3)
        q, k, v = (torch.randn(B, H, N, d, generator=g) for _ in range(3))
        segs = position_segments(layout, N, world, rank)
        kern = bench.CountingKernels(_OracleForwardKernels)
        o, lse = ring_forward_dist(*(bench.position_tokens(t, segs) for t in (q, k, v)), N, layout, causal,
                                   kernels=kern)
        idx = np.concatenate([t0 + st * np.arange(n) for t0, st, n in segs])
        out[rank] = (idx, o.numpy(), lse.numpy(), kern.launches)
    finally:
        dist.destroy_process_group()


def test_ring_mode_plumbing_gloo():
    """Every rank's slice of the ring mode's output equals the definition on its tokens, and
    the launch count is one library call (the folding partial) per visited segment pair."""
    import numpy as np

    import oracle
    from sequence_softmax_b200.ring_dist import position_segments, segment_in_future

    for world, layout, causal in [(2, "zigzag", True), (3, "striped", True), (2, "contiguous", False)]:
        out = mp.get_context("spawn").Manager().dict()
        port = 29800 + 11 * world + os.getpid() % 300
        mp.spawn(_ring_main, args=(world, port, layout, causal, out), nprocs=world, join=True)
        B, H, N, d = 1, 2, 16 * world, 8
        g = torch.Generator().manual_seed(3)
        q, k, v = (torch.randn(B, H, N, d, generator=g).numpy() for _ in range(3))
        o_ref, l_ref = oracle.attention(q, k, v, d ** -0.5, causal)
        for r in range(world):
            idx, o, lse, launches = out[r]
            assert np.abs(o - o_ref[:, :, idx]).max() <= 1e-5
            assert np.abs(lse - l_ref[:, :, idx]).max() <= 1e-5
            pairs = sum(not (causal and segment_in_future(qs, ks))
                        for c in range(world) for ks in position_segments(layout, N, world, c)
                        for qs in position_segments(layout, N, world, r))
            assert launches == pairs
