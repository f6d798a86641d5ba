"""USP (Ulysses all-to-all + ring) with the library's kernels on the one GPU this suite gets:
world size 1, and two processes sharing cuda:0 through gloo as a 1 x 2 mesh (Ulysses only)
and a 2 x 1 mesh (ring only). Gathered outputs and gradients against the fp64 oracle."""

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

B, H, N, D = 1, 4, 2048, 128


def _worker(rank, world, port, R, U, layout, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from sequence_softmax_b200 import usp
        from sequence_softmax_b200.inputs import make_qkv
        torch.cuda.set_device(0)
        intra, inter = usp.usp_groups(R, U)
        q, k, v = make_qkv(B, H, N, D, torch.bfloat16, seed=31, device="cuda")
        do = make_qkv(B, H, N, D, torch.bfloat16, seed=32, device="cuda")[0]
        idx = torch.as_tensor(usp.device_tokens(layout, N, R, U, rank // U, rank % U), device="cuda")
        loc = [t[:, :, idx].contiguous() for t in (q, k, v, do)]
        o, lse = usp.usp_forward(loc[0], loc[1], loc[2], N, layout, causal, intra_group=intra, inter_group=inter)
        grads = usp.usp_backward(loc[0], loc[1], loc[2], o, loc[3], lse, N, layout, causal, intra_group=intra,
                                 inter_group=inter)
        torch.cuda.synchronize()
        out[rank] = (idx.cpu(), o.float().cpu(), lse.cpu(), [g.float().cpu() for g in grads])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("R,U,layout,causal", [(1, 1, "zigzag", True), (1, 2, "contiguous", True),
                                               (2, 1, "zigzag", True)])
def test_usp_on_gpu(cuda, R, U, layout, causal):
    import oracle
    from sequence_softmax_b200.inputs import make_qkv

    from .parity import compare, compare_grads

    world = R * U
    out = mp.get_context("spawn").Manager().dict()
    port = 29950 + 13 * world + R + os.getpid() % 300
    mp.spawn(_worker, args=(world, port, R, U, layout, causal, out), nprocs=world, join=True)
    q, k, v = make_qkv(B, H, N, D, torch.bfloat16, seed=31, device="cuda")
    do = make_qkv(B, H, N, D, torch.bfloat16, seed=32, device="cuda")[0]
    qn, kn, vn, don = (t.float().cpu().numpy() for t in (q, k, v, do))
    o_ref, l_ref = oracle.attention(qn, kn, vn, D ** -0.5, causal)
    g_ref = oracle.attention_backward(qn, kn, vn, don, D ** -0.5, causal)
    o_all, l_all = np.zeros_like(o_ref), np.zeros_like(l_ref)
    g_all = [np.zeros_like(r) for r in g_ref]
    for r in range(world):
        idx, o, lse, grads = out[r]
        idx = idx.numpy()
        o_all[:, :, idx], l_all[:, :, idx] = o.numpy(), lse.numpy()
        for full, g in zip(g_all, grads):
            full[:, :, idx] = g.numpy()
    compare(o_all, l_all, o_ref, l_ref, "bf16", f"usp {R}x{U}")
    compare_grads(g_all, g_ref, "bf16", f"usp backward {R}x{U}")
