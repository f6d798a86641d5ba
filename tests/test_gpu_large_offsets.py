"""Tensors past 2^32 elements: 264 heads x 131072 tokens x d = 128 (4.4e9 elements, 8.9 GB
per bf16 tensor), causal zig-zag over 16 positions.

The last head's rows start past element 2^32 of every tensor, so each address the kernels
form there (TMA coordinates, epilogue stores, lse and D reads, the merge-free ring walk)
has to be computed in 64 bits. The forward's O and lse and the ring backward's dQ are
checked on sampled rows of the first and the last head against the oracle; dK and dV on
every head by the identities that hold at any size (each row of dS sums to zero, so the
keys' dK sum to zero; each row of P sums to one, so the keys' dV sum to the queries' dO).
"""

import numpy as np
import pytest
import torch

import oracle
from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import make_qkv, sample_rows

from .parity import compare, compare_grads

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

B, H, N, D, P, LAYOUT = 1, 264, 131072, 128, 16, "zigzag"
SCALE = D ** -0.5
GB = 1 << 30


def _head(t, h):
    return t[0, h].float().cpu().numpy()[None, None]


def test_forward_and_backward_past_2_32_elements(cuda):
    free, _ = torch.cuda.mem_get_info()
    if free < 96 * GB:
        pytest.skip(f"needs ~80 GB of device memory, {free / GB:.0f} GB free")
    q, k, v = make_qkv(B, H, N, D, torch.bfloat16, seed=11, device="cuda")
    assert (H - 1) * N * D > 2 ** 32  # the last head starts past element 2^32
    o, lse = binding.ring_forward(q, k, v, P, True, LAYOUT)
    assert binding.get_device_error() == binding.RA_OK

    rows = sample_rows(N, P, LAYOUT, count=256, seed=3)
    for h in (0, H - 1):
        qh, kh, vh = _head(q, h), _head(k, h), _head(v, h)
        o_ref, lse_ref = oracle.attention(qh, kh, vh, SCALE, True, rows=rows, row_block=32)
        compare(o[0, h].float().cpu().numpy()[rows], lse[0, h].cpu().numpy()[rows], o_ref[0, 0], lse_ref[0, 0],
                "bf16", f"forward head {h}")

    do = make_qkv(B, H, N, D, torch.bfloat16, seed=12, device="cuda")[0]
    dq, dk, dv = binding.ring_backward(q, k, v, o, do, lse, P, True, LAYOUT)
    assert binding.get_device_error() == binding.RA_OK

    qrows = rows[:128]
    for h in (0, H - 1):
        ref_q, _, _ = oracle.backward_rows(_head(q, h), _head(k, h), _head(v, h), _head(do, h), SCALE, True, qrows, [],
                                           heads=[(0, 0)])
        compare_grads([dq[0, h].float().cpu().numpy()[qrows][None]], [ref_q], "bf16", f"dQ rows head {h}")

    for h0 in range(0, H, 32):
        sl = slice(h0, h0 + 32)
        dk_sum = dk[:, sl].double().sum(dim=2)
        dk_abs = dk[:, sl].double().abs().sum(dim=2)
        assert torch.all(dk_sum.abs() <= 1e-2 * dk_abs + 1e-6), (h0, float((dk_sum.abs() / dk_abs).max()))
        dv_sum = dv[:, sl].double().sum(dim=2)
        do_sum = do[:, sl].double().sum(dim=2)
        dv_abs = dv[:, sl].double().abs().sum(dim=2)
        assert torch.all((dv_sum - do_sum).abs() <= 1e-2 * dv_abs + 1e-6), h0
