"""ra_ring_backward at the named long workloads, in the launch configuration the benchmark
times, against the fp64 oracle on sampled rows and on identities that hold at any size.

* seq32k-d128-causal-contig8: dQ on 256 sampled query rows (plus row 0, row N-1 and every
  chunk boundary) of two heads, and dK, dV on 128 sampled key rows of one head (the
  oracle computes that head's full forward state first).
* seq128k-d128-causal-zigzag16 (the benchmark's backward workload): dQ on sampled rows of
  two heads; dK, dV element by element on windows of key rows on both sides of every
  zig-zag chunk boundary (and at both ends of the sequence) of two heads, against the
  oracle's partial backward of every query row against the window (its forward state, O
  and lse of all 131072 rows of the head, is computed first by the forward oracle, row
  chunks in parallel threads); and, per head, the identities sum_j dK_j = 0 (every row of
  dS sums to zero: sum_j P_ij (dP_ij - D_i) = D_i - D_i) and sum_j dV_j = sum_i dO_i (every
  row of P sums to 1).
"""

import os
from concurrent.futures import ThreadPoolExecutor

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


def _forward_state(qh, kh, vh, scale, causal):
    """The forward oracle's O and lse for every row of one head [1, 1, N, d], computed in row
    chunks on parallel threads (one BLAS thread each: NumPy releases the GIL)."""
    from threadpoolctl import threadpool_limits

    N = qh.shape[2]
    chunks = np.array_split(np.arange(N), 128)
    workers = len(os.sched_getaffinity(0))
    with threadpool_limits(limits=1), ThreadPoolExecutor(workers) as ex:
        res = list(ex.map(lambda r: oracle.attention(qh, kh, vh, scale, causal, rows=r), chunks))
    return np.concatenate([o[0, 0] for o, _ in res]), np.concatenate([l[0, 0] for _, l in res])


def _check_dkdv_windows(w, q, k, v, do, dk, dv, h, half=4):
    """dK, dV of key rows b - half .. b + half - 1 around every chunk boundary b of the layout
    (and the first and last rows of the sequence), element by element against the oracle."""
    qh, kh, vh, doh = (_np_head(t, 0, h)[None, None] for t in (q, k, v, do))
    o_ref, lse_ref = _forward_state(qh, kh, vh, w.scale, w.causal)
    d_ref = oracle.delta(o_ref, doh[0, 0])
    parts = 2 * w.n_chunks if w.layout == "zigzag" else w.n_chunks
    c = w.N // parts
    starts = [0] + [b * c - half for b in range(1, parts)] + [w.N - 2 * half]
    got_k, got_v, ref_k, ref_v = [], [], [], []
    dk_h, dv_h = _np_head(dk, 0, h), _np_head(dv, 0, h)
    for j0 in starts:
        sl = slice(j0, j0 + 2 * half)
        _, rk, rv = oracle.partial_backward(qh, kh[:, :, sl], vh[:, :, sl], doh, lse_ref[None, None],
                                            d_ref[None, None], w.scale, w.causal, q_tok0=0, q_tok_stride=1,
                                            k_tok0=j0, k_tok_stride=1)
        ref_k.append(rk[0, 0])
        ref_v.append(rv[0, 0])
        got_k.append(dk_h[sl])
        got_v.append(dv_h[sl])
    none = np.zeros((0,))  # no dQ in this comparison
    compare_grads([none, np.concatenate(got_k), np.concatenate(got_v)],
                  [none, np.concatenate(ref_k), np.concatenate(ref_v)], "bf16",
                  f"{w.name} head {h} dK/dV at the chunk boundaries")


def test_backward_seq128k_zigzag(cuda):
    w, q, k, v, do, dq, dk, dv = _run("seq128k-d128-causal-zigzag16")
    rows = sample_rows(w.N, w.n_chunks, w.layout, count=128, seed=9)
    _check_dq_rows(w, q, k, v, do, dq, [(0, 3), (0, 30)], rows)
    for h in (3, 30):
        _check_dkdv_windows(w, q, k, v, do, dk, dv, h)
    dk64 = dk.double().sum(dim=2)                 # [B, H, d]
    dk_abs = dk.double().abs().sum(dim=2)
    assert torch.all(dk64.abs() <= 1e-2 * dk_abs + 1e-6), float((dk64.abs() / dk_abs).max())
    dv64 = dv.double().sum(dim=2)
    do64 = do.double().sum(dim=2)
    dv_abs = dv.double().abs().sum(dim=2)
    assert torch.all((dv64 - do64).abs() <= 1e-2 * dv_abs + 1e-6), float(((dv64 - do64).abs() / dv_abs).max())
