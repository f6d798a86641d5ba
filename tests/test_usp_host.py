"""USP (Ulysses all-to-all inside an intra group, the ring across inter groups) on gloo ranks
with CPU tensors: the token placement, the seq <-> head all-to-alls and the whole forward and
backward, with the library's kernels replaced by oracle-backed stand-ins, against the
definition."""

import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sequence_softmax_b200 import ring_dist, usp

from .test_peer_ring_host import _SharedPool


class _OracleKernels:
    """CPU stand-ins for partial_fold / partial / merge / backward_delta / partial_backward (fp64 oracle)."""

    @staticmethod
    def partial_fold(q, k, v, o_state, lse_state, causal=False, scale=None, q_tok0=0, q_tok_stride=1, k_tok0=0,
                     k_tok_stride=1, k_norm_max=None):
        import numpy as np

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
        return out, lse

    @staticmethod
    def merge(o_parts, lse_parts, out_dtype=torch.float32):
        import oracle
        o, l = oracle.merge(o_parts.numpy(), lse_parts.numpy())
        return torch.from_numpy(o).to(out_dtype), torch.from_numpy(l).float()

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


def _problem(R, U):
    B, H, N, d = 1, 2 * U, 8 * R * U * 2, 8
    r = np.random.default_rng(9)
    return [r.standard_normal((B, H, N, d)).astype(np.float32) for _ in range(4)]


def _main(rank, world, port, R, U, layout, causal, out, ring="message", pools=None):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        intra, inter = usp.usp_groups(R, U)
        q, k, v, do = _problem(R, U)
        N = q.shape[2]
        idx = usp.device_tokens(layout, N, R, U, rank // U, rank % U)
        loc = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, :, idx]))  # noqa: E731
        # the all-to-alls alone: seq -> head -> seq is the identity, and seq -> head gives this
        # member's head group over position r's tokens
        x = loc(q)
        xh = usp.seq_to_head(x, intra)
        pos = np.concatenate([t0 + st * np.arange(n)
                              for t0, st, n in ring_dist.position_segments(layout, N, R, rank // U)])
        hg = (rank % U) * (q.shape[1] // U)
        assert np.array_equal(xh.numpy(), q[:, hg:hg + q.shape[1] // U][:, :, pos])
        assert torch.equal(usp.head_to_seq(xh, intra), x)
        # peer ring: the ranks of inter group u share pools[u] as their peer memory
        share = _SharedPool(pools[rank % U]) if ring == "peer" else None
        o, lse = usp.usp_forward(loc(q), loc(k), loc(v), N, layout, causal, intra_group=intra, inter_group=inter,
                                 kernels=_OracleKernels, ring=ring, share=share)
        grads = usp.usp_backward(loc(q), loc(k), loc(v), o, loc(do), lse, N, layout, causal, intra_group=intra,
                                 inter_group=inter, kernels=_OracleKernels, ring=ring, share=share)
        out[rank] = (idx, o.numpy(), lse.numpy(), [g.numpy() for g in grads])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("R,U,layout,causal,ring", [(2, 2, "zigzag", True, "message"),
                                                    (1, 2, "contiguous", True, "message"),
                                                    (2, 1, "striped", True, "message"),
                                                    (2, 2, "contiguous", False, "message"),
                                                    (2, 2, "zigzag", True, "peer"),
                                                    (3, 1, "striped", True, "peer")])
def test_usp_matches_definition(R, U, layout, causal, ring):
    import oracle
    world = R * U
    pools = None
    if ring == "peer":
        q, *_ = _problem(R, U)
        B, H, N, d = q.shape
        nseg = len(ring_dist.position_segments(layout, N, R, 0))
        shp = (2, nseg, B, H // U, N // R // nseg, d)
        # per inter group: share calls forward K||V, backward K||V, backward accumulators
        pools = [[[torch.zeros(shp).share_memory_() for _ in range(R)] for _ in range(3)] for _ in range(U)]
    out = mp.get_context("spawn").Manager().dict()
    port = 29900 + 11 * world + 3 * R + (50 if ring == "peer" else 0) + os.getpid() % 300
    mp.spawn(_main, args=(world, port, R, U, layout, causal, out, ring, pools), nprocs=world, join=True)
    q, k, v, do = _problem(R, U)
    d = q.shape[-1]
    o_ref, l_ref = oracle.attention(q, k, v, d ** -0.5, causal)
    g_ref = oracle.attention_backward(q, k, v, do, d ** -0.5, causal)
    seen = np.zeros(q.shape[2], dtype=int)
    for rk in range(world):
        idx, o, lse, grads = out[rk]
        seen[idx] += 1
        assert np.abs(o - o_ref[:, :, idx]).max() <= 1e-5
        assert np.abs(lse - l_ref[:, :, idx]).max() <= 1e-5
        for g, r in zip(grads, g_ref):
            assert np.abs(g - r[:, :, idx]).max() <= 1e-4 * max(1.0, np.abs(r).max())
    assert np.all(seen == 1)  # every token on exactly one device
