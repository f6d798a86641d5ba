"""Split-KV use of the boundary: a few query rows at the end of a long sequence attend to
many KV chunks, each chunk's partial state comes from ra_partial and the states are combined
by ra_merge -- the lse associativity of the lecture 013 notes applied across chunks. Checked
against the fp64 oracle's causal attention on the same rows."""

import numpy as np
import pytest
import torch

import oracle
from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import make_qkv

from .parity import compare, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Lq,N,chunks,d", [(64, 65536, 16, 128), (16, 20000, 7, 64), (1, 4096, 4, 128)])
def test_decode_rows_over_many_chunks(cuda, Lq, N, chunks, d):
    B, H = 1, 4
    q_all, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=N + Lq, device="cuda")
    q = q_all[:, :, N - Lq:].contiguous()           # the last Lq tokens
    bounds = np.linspace(0, N, chunks + 1).astype(int)
    parts_o, parts_l = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        o_p, l_p = binding.partial(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(), causal=True,
                                   q_tok0=N - Lq, q_tok_stride=1, k_tok0=int(a), k_tok_stride=1)
        parts_o.append(o_p)
        parts_l.append(l_p)
    out, L = binding.merge(torch.stack(parts_o), torch.stack(parts_l), out_dtype=torch.float32)
    assert binding.get_device_error() == binding.RA_OK
    rows = np.arange(N - Lq, N)
    o_ref, l_ref = oracle.attention(to_np(q_all), to_np(k), to_np(v), d ** -0.5, True, rows=rows)
    compare(to_np(out), to_np(L), o_ref, l_ref, "bf16", f"split-KV Lq={Lq} N={N}")


def test_strided_chunks_merge(cuda):
    """Queries of one striped position against every striped position's keys."""
    B, H, N, d, P = 1, 2, 8192, 128, 8
    q_all, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=77, device="cuda")
    pq = 5
    q = q_all[:, :, pq::P].contiguous()
    parts_o, parts_l = [], []
    for pk in range(P):
        o_p, l_p = binding.partial(q, k[:, :, pk::P].contiguous(), v[:, :, pk::P].contiguous(), causal=True,
                                   q_tok0=pq, q_tok_stride=P, k_tok0=pk, k_tok_stride=P)
        parts_o.append(o_p)
        parts_l.append(l_p)
    out, L = binding.merge(torch.stack(parts_o), torch.stack(parts_l), out_dtype=torch.bfloat16)
    rows = np.arange(pq, N, P)
    o_ref, l_ref = oracle.attention(to_np(q_all), to_np(k), to_np(v), d ** -0.5, True, rows=rows)
    compare(to_np(out), to_np(L), o_ref, l_ref, "bf16", "striped merge")
