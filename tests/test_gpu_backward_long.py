"""ra_ring_backward at the named long workloads, in the launch configuration the benchmark
times, against the fp64 oracle on sampled rows and on identities that hold at any size.

* seq32k-d128-causal-contig8: dQ on 256 sampled query rows (plus row 0, row N-1 and every
  chunk boundary) of two heads, and dK, dV on 128 sampled key rows of one head (the
  oracle computes that head's full forward state first).
* seq128k-d128-causal-zigzag16 (the benchmark's backward workload): dQ on sampled rows of
  two heads, and per head the identities sum_j dK_j = 0 (every row of dS sums to zero:
  sum_j P_ij (dP_ij - D_i) = D_i - D_i) and sum_j dV_j = sum_i dO_i (every row of P sums to 1).
"""

import numpy as np
import pytest
import torch

import oracle
from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import WORKLOADS, make_qkv, sample_rows, workload_qkv

from .parity import compare_grads

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _run(name):
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w, device="cuda")
    do = make_qkv(w.B, w.H, w.N, w.d, w.torch_dtype, seed=1000, device="cuda")[0]
    o, lse = binding.ring_forward(q, k, v, w.n_chunks, w.causal, w.layout)
    dq, dk, dv = binding.ring_backward(q, k, v, o, do, lse, w.n_chunks, w.causal, w.layout)
    assert binding.get_device_error() == binding.RA_OK
    return w, q, k, v, do, dq, dk, dv


def _np_head(t, b, h):
    return t[b, h].float().cpu().numpy()


def _check_dq_rows(w, q, k, v, do, dq, heads, rows):
    qn, kn, vn, don = (np.stack([np.stack([_np_head(t, b, h) for (b, h) in heads])]) for t in (q, k, v, do))
    # the oracle sees the heads as a [1, len(heads), N, d] problem
    ref_q, _, _ = oracle.backward_rows(qn, kn, vn, don, w.scale, w.causal, rows, [],
                                       heads=[(0, i) for i in range(len(heads))])
    got = np.stack([_np_head(dq, b, h)[rows] for (b, h) in heads])
    compare_grads([got], [ref_q], "bf16", f"{w.name} dQ rows")


def test_backward_seq32k(cuda):
    w, q, k, v, do, dq, dk, dv = _run("seq32k-d128-causal-contig8")
    rows = sample_rows(w.N, w.n_chunks, w.layout, count=256, seed=7)
    _check_dq_rows(w, q, k, v, do, dq, [(0, 0), (0, 17)], rows)
    krows = sample_rows(w.N, w.n_chunks, w.layout, count=128, seed=8)
    h = 5
    qn, kn, vn, don = (_np_head(t, 0, h)[None, None] for t in (q, k, v, do))
    _, ref_k, ref_v = oracle.backward_rows(qn, kn, vn, don, w.scale, w.causal, [0], krows, heads=[(0, 0)])
    compare_grads([_np_head(dk, 0, h)[krows][None], _np_head(dv, 0, h)[krows][None]], [ref_k, ref_v], "bf16",
                  f"{w.name} dK/dV rows")


def test_backward_seq128k_zigzag(cuda):
    w, q, k, v, do, dq, dk, dv = _run("seq128k-d128-causal-zigzag16")
    rows = sample_rows(w.N, w.n_chunks, w.layout, count=128, seed=9)
    _check_dq_rows(w, q, k, v, do, dq, [(0, 3), (0, 30)], rows)
    dk64 = dk.double().sum(dim=2)                 # [B, H, d]
    dk_abs = dk.double().abs().sum(dim=2)
    assert torch.all(dk64.abs() <= 1e-2 * dk_abs + 1e-6), float((dk64.abs() / dk_abs).max())
    dv64 = dv.double().sum(dim=2)
    do64 = do.double().sum(dim=2)
    dv_abs = dv.double().abs().sum(dim=2)
    assert torch.all((dv64 - do64).abs() <= 1e-2 * dv_abs + 1e-6), float(((dv64 - do64).abs() / dv_abs).max())
