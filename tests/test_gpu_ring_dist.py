"""The multi-GPU ring (``ring_dist.ring_forward_dist`` / ``ring_backward_dist``) on the one GPU
this suite gets.

World size 1 runs the ring in one process. World size 2 runs two processes that share
cuda:0 and exchange K||V through a gloo group (host-staged): their kernels never wait on
one another, only the host exchange orders them. Results are gathered and compared with
the fp64 oracle.
"""

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

CASES = [("contiguous", True), ("zigzag", True), ("striped", True), ("contiguous", False)]


def _local_tokens(layout, N, W, r):
    from sequence_softmax_b200 import ring_dist
    return np.concatenate([t0 + st * np.arange(n) for t0, st, n in ring_dist.position_segments(layout, N, W, r)])


def _worker(rank, world, port, layout, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from sequence_softmax_b200 import ring_dist
        from sequence_softmax_b200.inputs import make_qkv
        torch.cuda.set_device(0)
        B, H, N, d = 1, 2, 2048, 128
        q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=11, device="cuda")
        idx = torch.as_tensor(_local_tokens(layout, N, world, rank), device="cuda")
        o, lse = ring_dist.ring_forward_dist(q[:, :, idx].contiguous(), k[:, :, idx].contiguous(),
                                             v[:, :, idx].contiguous(), N, layout, causal)
        torch.cuda.synchronize()
        out[rank] = (o.float().cpu(), lse.cpu(), idx.cpu())
    finally:
        dist.destroy_process_group()


def _run(world, layout, causal):
    import oracle
    from sequence_softmax_b200.inputs import make_qkv

    from .parity import compare

    out = mp.get_context("spawn").Manager().dict()
    port = 29700 + world * 10 + os.getpid() % 500
    mp.spawn(_worker, args=(world, port, layout, causal, out), nprocs=world, join=True)
    q, k, v = make_qkv(1, 2, 2048, 128, torch.bfloat16, seed=11, device="cuda")
    qn, kn, vn = (t.float().cpu().numpy() for t in (q, k, v))
    o_ref, l_ref = oracle.attention(qn, kn, vn, 128 ** -0.5, causal)
    for r in range(world):
        o, lse, idx = out[r]
        idx = idx.numpy()
        compare(o.numpy(), lse.numpy(), o_ref[:, :, idx], l_ref[:, :, idx], "bf16", f"rank {r} {layout}")


@pytest.mark.parametrize("layout,causal", CASES)
def test_ring_dist_world1(cuda, layout, causal):
    _run(1, layout, causal)


@pytest.mark.parametrize("layout,causal", CASES)
def test_ring_dist_world2_shared_gpu(cuda, layout, causal):
    _run(2, layout, causal)


def _bwd_worker(rank, world, port, layout, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from sequence_softmax_b200 import ring_dist
        from sequence_softmax_b200.inputs import make_qkv
        torch.cuda.set_device(0)
        B, H, N, d = 1, 2, 2048, 128
        q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=11, device="cuda")
        do = make_qkv(B, H, N, d, torch.bfloat16, seed=12, device="cuda")[0]
        idx = torch.as_tensor(_local_tokens(layout, N, world, rank), device="cuda")
        loc = [t[:, :, idx].contiguous() for t in (q, k, v, do)]
        o, lse = ring_dist.ring_forward_dist(loc[0], loc[1], loc[2], N, layout, causal)
        grads = ring_dist.ring_backward_dist(loc[0], loc[1], loc[2], o, loc[3], lse, N, layout, causal)
        torch.cuda.synchronize()
        out[rank] = ([g.float().cpu() for g in grads], idx.cpu())
    finally:
        dist.destroy_process_group()


def _run_bwd(world, layout, causal):
    import oracle
    from sequence_softmax_b200.inputs import make_qkv

    from .parity import compare_grads

    out = mp.get_context("spawn").Manager().dict()
    port = 29800 + world * 10 + os.getpid() % 500
    mp.spawn(_bwd_worker, args=(world, port, layout, causal, out), nprocs=world, join=True)
    q, k, v = make_qkv(1, 2, 2048, 128, torch.bfloat16, seed=11, device="cuda")
    do = make_qkv(1, 2, 2048, 128, torch.bfloat16, seed=12, device="cuda")[0]
    qn, kn, vn, don = (t.float().cpu().numpy() for t in (q, k, v, do))
    ref = oracle.attention_backward(qn, kn, vn, don, 128 ** -0.5, causal)
    got = [np.zeros_like(r) for r in ref]
    for r in range(world):
        grads, idx = out[r]
        idx = idx.numpy()
        for full, g in zip(got, grads):
            full[:, :, idx] = g.numpy()
    compare_grads(got, ref, "bf16", f"ring backward {layout} world {world}")


@pytest.mark.parametrize("layout,causal", [("zigzag", True), ("contiguous", False)])
def test_ring_backward_dist_world1(cuda, layout, causal):
    _run_bwd(1, layout, causal)


@pytest.mark.parametrize("layout,causal", [("zigzag", True), ("striped", True), ("contiguous", True)])
def test_ring_backward_dist_world2_shared_gpu(cuda, layout, causal):
    _run_bwd(2, layout, causal)
