"""ra_ring_forward on the GPU against the fp64 oracle, through the C-ABI.

Small and medium sizes are compared element by element; they span several 128-row tiles
and ragged tails. The named long workloads (32K, 128K and 1M tokens) are run in the launch
configuration the benchmark times and checked on 4096 seeded random query rows per head
plus row 0, row N-1 and every chunk boundary.
"""

import numpy as np
import pytest
import torch

import oracle
from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import WORKLOADS, make_qkv, ramp_qkv, sample_rows, workload_qkv

from .parity import compare, to_np

pytestmark = pytest.mark.gpu


def test_toy_workload_fp32(cuda):
    """The glossary's 4-device toy (seq 32, 4 chunks of 8, d 16, fp32): within 1e-5."""
    w = WORKLOADS["toy-4dev-seq32-d16"]
    q, k, v = workload_qkv(w, device="cuda")
    o, lse = binding.ring_forward(q, k, v, w.n_chunks, w.causal, w.layout)
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), w.scale, w.causal)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, "f32", w.name)
    full = torch.softmax(q[0, 0].cpu() @ k[0, 0].cpu().T / 4.0, dim=-1) @ v[0, 0].cpu()
    assert torch.allclose(o[0, 0].cpu(), full, atol=1e-5)  # the page's own check


SMALL = [
    # dtype, B, H, N, d, P, layout, causal
    ("f32", 1, 2, 200, 64, 4, "contiguous", True),
    ("f32", 2, 1, 96, 128, 3, "striped", True),
    ("f32", 1, 1, 120, 40, 3, "zigzag", True),
    ("f32", 1, 2, 128, 16, 2, "contiguous", False),
    ("bf16", 1, 2, 1024, 128, 4, "contiguous", False),
    ("bf16", 1, 2, 1024, 128, 4, "contiguous", True),
    ("bf16", 2, 1, 1024, 64, 4, "striped", True),
    ("bf16", 1, 2, 2048, 128, 4, "zigzag", True),
    ("bf16", 1, 2, 1000, 128, 4, "contiguous", True),   # 250-row chunks: ragged tiles
    ("bf16", 1, 1, 1000, 64, 4, "zigzag", True),        # 125-row chunks
    ("bf16", 1, 2, 1000, 128, 4, "striped", True),      # 250 rows per position, strided
    ("bf16", 1, 1, 1000, 128, 5, "striped", False),
    ("bf16", 1, 1, 130, 128, 1, "contiguous", True),    # one chunk = plain causal attention
    ("bf16", 1, 1, 1, 128, 1, "contiguous", True),      # a single token
    ("bf16", 1, 2, 4096, 128, 16, "zigzag", True),
    ("bf16", 1, 2, 4096, 128, 16, "striped", True),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
def test_ring_matches_oracle(cuda, case):
    kind, B, H, N, d, P, layout, causal = case
    dtype = torch.float32 if kind == "f32" else torch.bfloat16
    q, k, v = make_qkv(B, H, N, d, dtype, seed=N + P, device="cuda")
    o, lse = binding.ring_forward(q, k, v, P, causal, layout)
    assert binding.get_device_error() == binding.RA_OK
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), d ** -0.5, causal)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, kind, str(case))


RAMP_CASES = [
    # jump (log2 units per block), block (keys), N, d, P, layout, causal
    (10.0, 128, 1024, 128, 1, "contiguous", False),  # the running max moves past the threshold every tile
    (6.0, 128, 1024, 128, 1, "contiguous", True),    # moves by less than the threshold, then past it
    (10.0, 128, 1024, 64, 1, "contiguous", True),
    (10.0, 128, 2048, 128, 4, "contiguous", False),  # ring order: a big jump when the walk wraps
    (10.0, 128, 2048, 128, 4, "zigzag", True),
    (6.0, 128, 2048, 128, 4, "striped", True),
    (10.0, 64, 1024, 128, 1, "contiguous", False),   # jumps in both halves of every tile
    (10.0, 64, 2048, 128, 4, "zigzag", True),
    (10.0, 64, 1024, 64, 1, "contiguous", True),
    (80.0, 64, 1024, 128, 1, "contiguous", False),   # a second half far past the running max
    (80.0, 64, 2048, 128, 4, "zigzag", True),
    (80.0, 64, 1024, 64, 2, "striped", True),
]


@pytest.mark.parametrize("case", RAMP_CASES, ids=lambda c: "-".join(map(str, c)))
def test_running_max_rescale_matches_oracle(cuda, case):
    """Scores that rise block after block (the score ramp of the inputs module) make the
    forward move its running maximum, and rescale O and l, while it walks the keys: at tile
    starts (128-key blocks), in the middle of tiles too (64-key blocks), and by far more than
    the threshold within a tile's second half (jumps of 80 log2 units)."""
    jump, block, N, d, P, layout, causal = case
    q, k, v = ramp_qkv(N, d, jump, seed=N + P, device="cuda", block=block)
    o, lse = binding.ring_forward(q, k, v, P, causal, layout)
    assert binding.get_device_error() == binding.RA_OK
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), d ** -0.5, causal)
    assert np.abs(o_ref).mean() > 10 * 2e-3  # a wrong rescale moves O by far more than the mean tolerance
    compare(to_np(o), to_np(lse), o_ref, lse_ref, "bf16", str(case))


SKIP_CASES = [
    # jump (log2 units per 128-key block), N, d, P, layout, causal
    (2.5, 1024, 128, 1, "contiguous", False),  # bound within 24 of the first tile's max: m kept
    (2.5, 1024, 128, 1, "contiguous", True),
    (2.5, 1024, 64, 1, "contiguous", False),
    (2.5, 2048, 128, 2, "zigzag", True),       # a rise of 37.5: skipped and computed maxima mixed
    (2.5, 2048, 128, 1, "contiguous", False),
]


@pytest.mark.parametrize("case", SKIP_CASES, ids=lambda c: "-".join(map(str, c)))
def test_row_max_skip_matches_oracle(cuda, case):
    """Keys nearly parallel to the queries (the ramp with a small spread) make the key-norm
    bound tight: from the second tile on the forward keeps the first tile's max while the
    scores rise by up to 17.5 log2 units (exponentials up to ~2^17.5), and on the longer
    ramp it has to take the row max again part of the way."""
    jump, N, d, P, layout, causal = case
    q, k, v = ramp_qkv(N, d, jump, seed=N + d, device="cuda", spread=0.05)
    o, lse = binding.ring_forward(q, k, v, P, causal, layout)
    assert binding.get_device_error() == binding.RA_OK
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), d ** -0.5, causal)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, "bf16", str(case))
    # without lse the forward has no key bound and always takes the row max
    o2, _ = binding.ring_forward(q, k, v, P, causal, layout, return_lse=False)
    compare(to_np(o2), None, o_ref, None, "bf16", str(case) + " no lse")


@pytest.mark.parametrize("scale", [0.05, 0.3, 1.0])
def test_explicit_scale_matches_oracle(cuda, scale):
    """A softmax scale other than d^-1/2. At 0.05 the key-norm bound is ~11 log2 units and the
    row-max skip fires from the second tile; at 0.3 and 1.0 it is far above the scores (and
    at 1.0 each row's softmax is nearly one-hot), so every tile takes the max."""
    B, H, N, d, P = 1, 2, 2048, 128, 4
    q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=31, device="cuda")
    o, lse = binding.ring_forward(q, k, v, P, True, "zigzag", scale=scale)
    assert binding.get_device_error() == binding.RA_OK
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), scale, True)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, "bf16", f"scale {scale}")


def test_layout_invariance_on_gpu(cuda):
    """Contiguous, striped and zig-zag give the same attention (the layout moves work only)."""
    B, H, N, d, P = 1, 4, 4096, 128, 8
    q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=21, device="cuda")
    outs = [binding.ring_forward(q, k, v, P, True, lay) for lay in ("contiguous", "striped", "zigzag")]
    for o, l in outs[1:]:
        assert (o.float() - outs[0][0].float()).abs().max().item() <= 2e-2
        assert (l - outs[0][1]).abs().max().item() <= 1e-2


def test_deterministic(cuda):
    q, k, v = make_qkv(1, 2, 2048, 128, torch.bfloat16, seed=5, device="cuda")
    a, la = binding.ring_forward(q, k, v, 4, True, "zigzag")
    b, lb = binding.ring_forward(q, k, v, 4, True, "zigzag")
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_host_buffers_round_trip(cuda):
    """Host (pinned) tensors in, host tensors out: the end-to-end path of the public call."""
    q, k, v = make_qkv(1, 2, 1024, 128, torch.bfloat16, seed=8, device="cpu")
    q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o, lse = binding.ring_forward(q, k, v, 4, True, "contiguous")
    assert o.device.type == "cpu" and lse.device.type == "cpu"
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), 128 ** -0.5, True)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, "bf16", "host buffers")


@pytest.mark.parametrize("pinned", [True, False])
def test_host_pipeline_equals_device_call(cuda, pinned):
    """The host path runs the (batch, head) rows in groups with copies overlapped; heads are
    independent, so it must equal one device call bit for bit (6 rows in 4 uneven groups)."""
    q, k, v = make_qkv(2, 3, 1024, 128, torch.bfloat16, seed=18, device="cpu")
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o_h, l_h = binding.ring_forward(q, k, v, 4, True, "zigzag")
    o_d, l_d = binding.ring_forward(q.cuda(), k.cuda(), v.cuda(), 4, True, "zigzag")
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())


@pytest.mark.parametrize("name", ["seq4k-d64-noncausal-8chunks", "seq4k-d64-noncausal-8chunks-qx4"])
def test_workload_full_compare(cuda, name):
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w, device="cuda")
    o, lse = binding.ring_forward(q, k, v, w.n_chunks, w.causal, w.layout)
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), w.scale, w.causal)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, "bf16", name)


LONG = ["seq32k-d128-causal-contig8", "seq128k-d128-causal-zigzag16", "seq128k-d128-causal-striped16",
        "seq1m-d128-causal-zigzag16"]


def _oracle_rows_per_head(qs, k, v, rows, w, threads=4):
    """Oracle on sampled rows, one head per worker thread (NumPy releases the GIL)."""
    from concurrent.futures import ThreadPoolExecutor

    def one(h):
        full_q = np.zeros((1, 1, w.N, w.d), dtype=np.float32)  # calloc: only sampled rows are touched
        full_q[0, 0, rows] = qs[0, h]
        kh = to_np(k[:, h:h + 1])
        vh = to_np(v[:, h:h + 1])
        oh, lh = oracle.attention(full_q, kh, vh, w.scale, w.causal, rows=rows, row_block=32)
        return oh[0, 0], lh[0, 0]

    o_ref = np.zeros((w.B, w.H, len(rows), w.d))
    lse_ref = np.zeros((w.B, w.H, len(rows)))
    with ThreadPoolExecutor(threads) as ex:
        for h, (oh, lh) in enumerate(ex.map(one, range(w.H))):
            o_ref[0, h], lse_ref[0, h] = oh, lh
    return o_ref, lse_ref


@pytest.mark.slow
@pytest.mark.parametrize("name", LONG)
def test_workload_sampled_rows(cuda, name):
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w, device="cuda")
    o, lse = binding.ring_forward(q, k, v, w.n_chunks, w.causal, w.layout)
    assert binding.get_device_error() == binding.RA_OK
    rows = sample_rows(w.N, w.n_chunks, w.layout)
    ridx = torch.as_tensor(rows, device="cuda")
    qs = to_np(q[:, :, ridx])
    o_ref, lse_ref = _oracle_rows_per_head(qs, k, v, rows, w)
    stats = compare(to_np(o[:, :, ridx]), to_np(lse[:, :, ridx]), o_ref, lse_ref, "bf16", name)
    print(name, stats)


def test_more_heads_than_a_grid_dimension(cuda):
    """65540 heads (B * H beyond 65535): the key-bound passes run one-dimensional grids, so the
    forward keeps its row-max skip and ra_key_norm_max serves any head count. Sampled heads
    against the oracle, every head's key bound against torch's norms."""
    B, H, N, d, P = 2, 32770, 256, 64, 2
    q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=41, device="cuda")
    o, lse = binding.ring_forward(q, k, v, P, True, "zigzag")
    assert binding.get_device_error() == binding.RA_OK
    for b, h in ((0, 0), (0, 32769), (1, 0), (1, 16384), (1, 32769)):
        o_ref, lse_ref = oracle.attention(to_np(q[b:b + 1, h:h + 1]), to_np(k[b:b + 1, h:h + 1]),
                                          to_np(v[b:b + 1, h:h + 1]), d ** -0.5, True)
        compare(to_np(o[b:b + 1, h:h + 1]), to_np(lse[b:b + 1, h:h + 1]), o_ref, lse_ref, "bf16", f"head {b},{h}")
    kmax = binding.key_norm_max(k)
    ref = k.float().norm(dim=-1).amax(dim=-1)
    assert torch.allclose(kmax, ref, rtol=1e-5, atol=0.0)
