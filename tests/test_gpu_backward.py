"""The backward pass on the GPU against the fp64 oracle, through the C-ABI.

ring_backward runs on the product chain (ring_forward's O and lse feed it); the oracle
recomputes everything from Q, K, V and dO. partial_backward gets the oracle's final lse and D
for its query rows (inputs flow from the oracle to the GPU, never back).
"""

import numpy as np
import pytest
import torch

import oracle
from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import make_qkv, ramp_qkv

from .parity import compare_grads, to_np

pytestmark = pytest.mark.gpu


def _upstream(B, H, N, d, dtype, seed):
    return make_qkv(B, H, N, d, dtype, seed=seed, device="cuda")[0]


RING_CASES = [
    # dtype, B, H, N, d, P, causal, layout
    ("f32", 1, 1, 32, 16, 4, False, "contiguous"),   # the 4-device toy's shape
    ("f32", 1, 2, 64, 32, 4, True, "striped"),
    ("f32", 2, 1, 48, 128, 3, True, "zigzag"),
    ("bf16", 1, 2, 1024, 128, 4, True, "zigzag"),
    ("bf16", 1, 2, 1024, 64, 4, True, "striped"),
    ("bf16", 2, 2, 768, 128, 3, True, "contiguous"),
    ("bf16", 1, 2, 768, 128, 4, True, "zigzag"),     # 96-token chunks: every tile ragged
    ("bf16", 1, 2, 512, 128, 2, False, "contiguous"),
    ("bf16", 1, 2, 640, 64, 5, False, "striped"),
    ("bf16", 1, 1, 200, 128, 1, True, "contiguous"),  # one ragged segment
    ("bf16", 1, 1, 128, 64, 1, True, "contiguous"),   # one tile
]


@pytest.mark.parametrize("case", RING_CASES, ids=lambda c: "-".join(map(str, c)))
def test_ring_backward_matches_oracle(cuda, case):
    kind, B, H, N, d, P, causal, layout = case
    dtype = torch.float32 if kind == "f32" else torch.bfloat16
    q, k, v = make_qkv(B, H, N, d, dtype, seed=N + P, device="cuda")
    do = _upstream(B, H, N, d, dtype, seed=N + P + 1000)
    o, lse = binding.ring_forward(q, k, v, P, causal, layout)
    dq, dk, dv = binding.ring_backward(q, k, v, o, do, lse, P, causal, layout)
    assert binding.get_device_error() == binding.RA_OK
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), d ** -0.5, causal)
    print(case, compare_grads((to_np(dq), to_np(dk), to_np(dv)), ref, kind, str(case)))


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_ring_backward_on_rising_scores(cuda, layout):
    """The score ramp (every 128-key block scores ~10 log2 units above the one before): the
    forward rescales its running state at every block and the backward rebuilds P from the
    final lse."""
    N, d, P = 1024, 128, 4
    q, k, v = ramp_qkv(N, d, 10.0, seed=7, device="cuda")
    do = _upstream(1, 1, N, d, torch.bfloat16, seed=8)
    o, lse = binding.ring_forward(q, k, v, P, True, layout)
    dq, dk, dv = binding.ring_backward(q, k, v, o, do, lse, P, True, layout)
    assert binding.get_device_error() == binding.RA_OK
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), d ** -0.5, True)
    print(layout, compare_grads((to_np(dq), to_np(dk), to_np(dv)), ref, "bf16", layout))


def test_ring_backward_layout_invariant(cuda):
    """The layout changes the order of the additions only."""
    B, H, N, d = 1, 2, 1024, 128
    q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=5, device="cuda")
    do = _upstream(B, H, N, d, torch.bfloat16, seed=6)
    o, lse = binding.ring_forward(q, k, v, 4, True, "contiguous")
    ref = [to_np(t) for t in binding.ring_backward(q, k, v, o, do, lse, 4, True, "contiguous")]
    for layout, P in (("striped", 4), ("zigzag", 4), ("zigzag", 2), ("contiguous", 1)):
        got = [to_np(t) for t in binding.ring_backward(q, k, v, o, do, lse, P, True, layout)]
        for g, r in zip(got, ref):
            assert np.abs(g - r).max() <= 1e-2 * np.abs(r).max(), layout


PARTIAL_CASES = [
    # dtype, B, H, Lq, Lk, d, causal, q_tok0, q_ts, k_tok0, k_ts
    ("f32", 1, 2, 40, 56, 16, True, 20, 1, 0, 1),
    ("f32", 1, 1, 33, 20, 128, False, 0, 1, 0, 1),
    ("bf16", 1, 2, 300, 200, 128, False, 0, 1, 0, 1),     # ragged tails on both sides
    ("bf16", 1, 2, 384, 256, 64, True, 256, 1, 0, 1),     # keys partly on the diagonal
    ("bf16", 2, 1, 256, 384, 128, True, 0, 1, 128, 1),    # keys partly in the future: empty rows
    ("bf16", 1, 2, 256, 256, 128, True, 3, 8, 5, 8),      # striped positions
    ("bf16", 1, 1, 1, 1, 128, False, 0, 1, 0, 1),         # one row, one key
]


@pytest.mark.parametrize("case", PARTIAL_CASES, ids=lambda c: "-".join(map(str, c)))
def test_partial_backward_matches_oracle(cuda, case):
    kind, B, H, Lq, Lk, d, causal, qt0, qts, kt0, kts = case
    dtype = torch.float32 if kind == "f32" else torch.bfloat16
    q, _, _ = make_qkv(B, H, Lq, d, dtype, seed=Lq + 7, device="cuda")
    _, k, v = make_qkv(B, H, Lk, d, dtype, seed=Lk + 9, device="cuda")
    do = _upstream(B, H, Lq, d, dtype, seed=Lq + Lk)
    scale = d ** -0.5
    # one chunk only: its partial state is the final state of these query rows
    o_ref, lse_ref = oracle.partial(to_np(q), to_np(k), to_np(v), scale, causal, qt0, qts, kt0, kts)
    lse_t = torch.tensor(lse_ref, dtype=torch.float32, device="cuda")
    d_t = torch.tensor(oracle.delta(o_ref, to_np(do)), dtype=torch.float32, device="cuda")
    acc = [torch.zeros(B, H, Lq, d, device="cuda"), torch.zeros(B, H, Lk, d, device="cuda"),
           torch.zeros(B, H, Lk, d, device="cuda")]
    binding.partial_backward(q, k, v, do, lse_t, d_t, *acc, causal=causal, scale=scale, q_tok0=qt0,
                             q_tok_stride=qts, k_tok0=kt0, k_tok_stride=kts)
    assert binding.get_device_error() == binding.RA_OK
    ref = oracle.partial_backward(to_np(q), to_np(k), to_np(v), to_np(do), to_np(lse_t), to_np(d_t), scale, causal,
                                  qt0, qts, kt0, kts)
    print(case, compare_grads([to_np(t) for t in acc], ref, kind, str(case)))


def test_partial_backward_accumulates_the_ring(cuda):
    """Every (query position, KV chunk) pair of a 4-way contiguous split, added into per-position
    accumulators, gives the full gradients (the multi-GPU ring's arithmetic in pieces)."""
    B, H, N, d, P = 1, 2, 1024, 128, 4
    c = N // P
    q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=21, device="cuda")
    do = _upstream(B, H, N, d, torch.bfloat16, seed=22)
    o, lse = binding.ring_forward(q, k, v, P, True, "contiguous")
    delta = binding.backward_delta(o, do)
    dq = [torch.zeros(B, H, c, d, device="cuda") for _ in range(P)]
    dk = [torch.zeros(B, H, c, d, device="cuda") for _ in range(P)]
    dv = [torch.zeros(B, H, c, d, device="cuda") for _ in range(P)]
    blk = lambda t, p: t[:, :, p * c:(p + 1) * c].contiguous()  # noqa: E731
    for pq in range(P):
        for s in range(P):
            pk = (pq - s) % P   # ring order
            if pk > pq:
                continue        # wholly in the future
            binding.partial_backward(blk(q, pq), blk(k, pk), blk(v, pk), blk(do, pq), blk(lse, pq), blk(delta, pq),
                                     dq[pq], dk[pk], dv[pk], causal=True, q_tok0=pq * c, k_tok0=pk * c)
    assert binding.get_device_error() == binding.RA_OK
    got = [to_np(torch.cat(x, dim=2)) for x in (dq, dk, dv)]
    ref = oracle.attention_backward(to_np(q), to_np(k), to_np(v), to_np(do), d ** -0.5, True)
    compare_grads(got, ref, "bf16", "partials")


def test_partial_backward_empty_keys_is_noop(cuda):
    q, _, _ = make_qkv(1, 1, 64, 128, torch.bfloat16, seed=3, device="cuda")
    k = torch.empty(1, 1, 0, 128, device="cuda", dtype=torch.bfloat16)
    z = torch.zeros(1, 1, 64, device="cuda")
    acc = [torch.full((1, 1, 64, 128), 2.0, device="cuda"), torch.zeros(1, 1, 0, 128, device="cuda"),
           torch.zeros(1, 1, 0, 128, device="cuda")]
    binding.partial_backward(q, k, k.clone(), q.clone(), z, z, *acc)
    assert torch.all(acc[0] == 2.0)


@pytest.mark.parametrize("kind,d", [("bf16", 128), ("bf16", 64), ("f32", 48)])
def test_backward_delta(cuda, kind, d):
    dtype = torch.float32 if kind == "f32" else torch.bfloat16
    o, do, _ = make_qkv(2, 3, 333, d, dtype, seed=d, device="cuda")
    got = to_np(binding.backward_delta(o, do))
    ref = oracle.delta(to_np(o), to_np(do))
    assert np.abs(got - ref).max() <= 1e-5 * (1 + np.abs(ref).max())


def test_ring_backward_is_deterministic(cuda):
    """Every row of dQ, dK and dV is produced by exactly one CTA (no reductions into shared
    memory between CTAs), so two runs agree bit for bit."""
    q, k, v = make_qkv(1, 4, 2048, 128, torch.bfloat16, seed=41, device="cuda")
    do = _upstream(1, 4, 2048, 128, torch.bfloat16, seed=42)
    o, lse = binding.ring_forward(q, k, v, 4, True, "zigzag")
    a = binding.ring_backward(q, k, v, o, do, lse, 4, True, "zigzag")
    b = binding.ring_backward(q, k, v, o, do, lse, 4, True, "zigzag")
    for x, y in zip(a, b):
        assert torch.equal(x, y)
