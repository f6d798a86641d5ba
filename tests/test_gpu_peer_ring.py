"""The peer-memory ring (``peer_ring``) on the one GPU this suite gets.

World size 1 runs in one process. World size 2 runs two processes that share cuda:0: each
maps the other's K||V (and, in the backward, dK||dV accumulator) buffers through CUDA IPC,
and the library's kernels read and accumulate through those mappings; gloo carries the
handles and the barriers between steps. Both ways of reading K||V run: "direct" (the
kernels read the owner's buffer through the mapping) and "copy" (each step's block is
pulled into a local double buffer one step ahead with one DMA copy on a copy stream, the
copy ordered after the kernels that last read that buffer). The kernels of the two
processes never wait on one another. Each rank's O, lse, dQ, dK and dV are compared with the fp64 oracle and must equal
``ring_dist``'s bit for bit (same kernels, same values, same order).
"""

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

B, H, N, D = 1, 2, 2048, 128


def _local_tokens(layout, W, r):
    from sequence_softmax_b200 import ring_dist
    return np.concatenate([t0 + st * np.arange(n) for t0, st, n in ring_dist.position_segments(layout, N, W, r)])


def _worker(rank, world, port, layout, causal, mode, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from sequence_softmax_b200 import peer_ring, ring_dist
        from sequence_softmax_b200.inputs import make_qkv
        torch.cuda.set_device(0)
        q, k, v = make_qkv(B, H, N, D, torch.bfloat16, seed=11, device="cuda")
        do = make_qkv(B, H, N, D, torch.bfloat16, seed=12, device="cuda")[0]
        idx = torch.as_tensor(_local_tokens(layout, world, rank), device="cuda")
        lq, lk, lv, ldo = (t[:, :, idx].contiguous() for t in (q, k, v, do))
        o, lse = peer_ring.ring_forward_peer(lq, lk, lv, N, layout, causal, mode=mode)
        grads = peer_ring.ring_backward_peer(lq, lk, lv, o, ldo, lse, N, layout, causal, mode=mode)
        o_d, lse_d = ring_dist.ring_forward_dist(lq, lk, lv, N, layout, causal)
        grads_d = ring_dist.ring_backward_dist(lq, lk, lv, o, ldo, lse, N, layout, causal)
        torch.cuda.synchronize()
        same = torch.equal(o, o_d) and torch.equal(lse, lse_d) and all(torch.equal(a, b) for a, b in zip(grads, grads_d))
        out[rank] = (o.float().cpu(), lse.cpu(), [g.float().cpu() for g in grads], idx.cpu(), same)
    finally:
        dist.destroy_process_group()


def _run(world, layout, causal, mode="copy"):
    import oracle
    from sequence_softmax_b200.inputs import make_qkv

    from .parity import compare, compare_grads

    out = mp.get_context("spawn").Manager().dict()
    port = 29900 + world * 10 + os.getpid() % 500
    mp.spawn(_worker, args=(world, port, layout, causal, mode, out), nprocs=world, join=True)
    q, k, v = make_qkv(B, H, N, D, torch.bfloat16, seed=11, device="cuda")
    do = make_qkv(B, H, N, D, torch.bfloat16, seed=12, device="cuda")[0]
    qn, kn, vn, don = (t.float().cpu().numpy() for t in (q, k, v, do))
    o_ref, l_ref = oracle.attention(qn, kn, vn, D ** -0.5, causal)
    g_ref = oracle.attention_backward(qn, kn, vn, don, D ** -0.5, causal)
    got = [np.zeros_like(r) for r in g_ref]
    for r in range(world):
        o, lse, grads, idx, same = out[r]
        idx = idx.numpy()
        assert same, f"rank {r}: peer ring ({mode}) differs from ring_dist"
        compare(o.numpy(), lse.numpy(), o_ref[:, :, idx], l_ref[:, :, idx], "bf16", f"rank {r} {layout}")
        for full, g in zip(got, grads):
            full[:, :, idx] = g.numpy()
    compare_grads(got, g_ref, "bf16", f"peer ring backward {layout} world {world}")


@pytest.mark.parametrize("layout,causal", [("zigzag", True), ("contiguous", False)])
def test_peer_ring_world1(cuda, layout, causal):
    _run(1, layout, causal)


@pytest.mark.parametrize("mode", ["copy", "direct"])
@pytest.mark.parametrize("layout,causal", [("zigzag", True), ("striped", True), ("contiguous", True),
                                           ("contiguous", False)])
def test_peer_ring_world2_shared_gpu(cuda, layout, causal, mode):
    _run(2, layout, causal, mode)
