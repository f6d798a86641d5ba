"""ra_partial on the GPU against the oracle's partial state (fp64), through the C-ABI."""

import numpy as np
import pytest
import torch

import oracle
from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import make_qkv

from .parity import compare, to_np

pytestmark = pytest.mark.gpu

CASES = [
    # dtype, B, H, Lq, Lk, d, causal, q_tok0, q_ts, k_tok0, k_ts
    ("f32", 1, 2, 64, 96, 16, False, 0, 1, 0, 1),
    ("f32", 2, 1, 70, 45, 128, True, 100, 1, 60, 1),      # ragged, partly visible
    ("f32", 1, 1, 40, 40, 33, True, 3, 4, 1, 4),          # striped positions
    ("bf16", 1, 2, 256, 256, 128, False, 0, 1, 0, 1),
    ("bf16", 2, 2, 384, 640, 64, False, 0, 1, 0, 1),
    ("bf16", 1, 3, 300, 333, 128, False, 0, 1, 0, 1),     # ragged tails on both sides
    ("bf16", 1, 2, 512, 512, 128, True, 512, 1, 0, 1),    # chunk wholly in the past: full
    ("bf16", 1, 2, 512, 512, 128, True, 0, 1, 0, 1),      # diagonal chunk
    ("bf16", 1, 2, 512, 512, 64, True, 0, 1, 256, 1),     # keys partly in the future, empty rows
    ("bf16", 1, 1, 256, 256, 128, True, 0, 1, 4096, 1),   # keys wholly in the future: all empty
    ("bf16", 1, 2, 256, 384, 128, True, 5, 16, 2, 16),    # striped query / key positions
    ("bf16", 1, 1, 1, 1, 128, False, 0, 1, 0, 1),         # one row, one key
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_partial_matches_oracle(cuda, case):
    kind, B, H, Lq, Lk, d, causal, qt0, qts, kt0, kts = case
    dtype = torch.float32 if kind == "f32" else torch.bfloat16
    q, _, _ = make_qkv(B, H, Lq, d, dtype, seed=Lq + Lk, device="cuda")
    _, k, v = make_qkv(B, H, Lk, d, dtype, seed=Lq * Lk + 1, device="cuda")
    o, lse = binding.partial(q, k, v, causal=causal, q_tok0=qt0, q_tok_stride=qts, k_tok0=kt0, k_tok_stride=kts)
    assert binding.get_device_error() == binding.RA_OK
    o_ref, lse_ref = oracle.partial(to_np(q), to_np(k), to_np(v), d ** -0.5, causal, qt0, qts, kt0, kts)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, kind, str(case))


def test_partial_empty_keys(cuda):
    q, _, _ = make_qkv(1, 2, 100, 128, torch.bfloat16, seed=1, device="cuda")
    k = torch.empty(1, 2, 0, 128, device="cuda", dtype=torch.bfloat16)
    o, lse = binding.partial(q, k, k.clone())
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_partials_merge_to_full_attention(cuda):
    """The ring's arithmetic in pieces: partial states of 4 KV chunks merged on the GPU equal
    full causal attention from the oracle."""
    B, H, N, d, P = 1, 2, 1024, 128, 4
    q, k, v = make_qkv(B, H, N, d, torch.bfloat16, seed=11, device="cuda")
    c = N // P
    parts_o, parts_l = [], []
    for p in range(P):
        o_p, l_p = binding.partial(q, k[:, :, p * c:(p + 1) * c].contiguous(), v[:, :, p * c:(p + 1) * c].contiguous(),
                                   causal=True, q_tok0=0, q_tok_stride=1, k_tok0=p * c, k_tok_stride=1)
        parts_o.append(o_p)
        parts_l.append(l_p)
    out, L = binding.merge(torch.stack(parts_o), torch.stack(parts_l), out_dtype=torch.bfloat16)
    o_ref, l_ref = oracle.attention(to_np(q), to_np(k), to_np(v), d ** -0.5, True)
    compare(to_np(out), to_np(L), o_ref, l_ref, "bf16", "partials+merge")


FOLD_CASES = [
    # dtype, B, H, Lq, Lk, d, causal, q_tok0, k_tok0, k_tok_stride
    ("bf16", 1, 2, 384, 256, 128, True, 0, 128, 1),      # query rows 0-127 see nothing of the chunk
    ("bf16", 2, 1, 300, 500, 64, False, 0, 0, 1),
    ("bf16", 1, 1, 256, 256, 128, True, 0, 3, 4),       # strided keys: striped positions
    ("f32", 1, 2, 70, 90, 32, True, 40, 10, 1),
]


@pytest.mark.parametrize("case", FOLD_CASES, ids=lambda c: "-".join(map(str, c)))
def test_partial_fold_equals_partial_then_merge(cuda, case):
    """ra_partial_fold leaves exactly (bit for bit) the state that ra_partial into a scratch
    state followed by ra_merge of [state, partial] (fp32 output) would: from the empty state,
    and from a state whose rows include empty ones (lse = -inf) and finite ones."""
    kind, B, H, Lq, Lk, d, causal, q_tok0, k_tok0, k_ts = case
    dtype = torch.float32 if kind == "f32" else torch.bfloat16
    q, k, v = make_qkv(B, H, Lq, d, dtype, seed=Lq + Lk, device="cuda", Nk=Lk)
    g = torch.Generator(device="cuda").manual_seed(7)
    starts = [
        (torch.zeros(B, H, Lq, d, device="cuda"), torch.full((B, H, Lq), float("-inf"), device="cuda")),
        (torch.randn(B, H, Lq, d, device="cuda", generator=g),
         torch.where(torch.rand(B, H, Lq, device="cuda", generator=g) < 0.2, float("-inf"),
                     torch.randn(B, H, Lq, device="cuda", generator=g) + 5.0)),
    ]
    kw = dict(causal=causal, q_tok0=q_tok0, k_tok0=k_tok0, k_tok_stride=k_ts)
    for o0, l0 in starts:
        o_p, l_p = binding.partial(q, k, v, **kw)
        want_o, want_l = binding.merge(torch.stack([o0, o_p]), torch.stack([l0, l_p]), out_dtype=torch.float32)
        st_o, st_l = o0.clone(), l0.clone()
        binding.partial_fold(q, k, v, st_o, st_l, **kw)
        assert binding.get_device_error() == binding.RA_OK
        assert torch.equal(st_o, want_o) and torch.equal(st_l, want_l)
    # an empty chunk leaves the state untouched
    st_o, st_l = starts[1][0].clone(), starts[1][1].clone()
    binding.partial_fold(q, k[:, :, :0].contiguous(), v[:, :, :0].contiguous(), st_o, st_l, **kw)
    torch.cuda.synchronize()
    assert torch.equal(st_o, starts[1][0]) and torch.equal(st_l, starts[1][1])


@pytest.mark.parametrize("d", [64, 128])
def test_key_norm_max_matches_the_norms(cuda, d):
    """ra_key_norm_max against fp64 norms of the same bf16 keys, for one to 70000 keys per
    head (one to 683 chunks per head): within fp32 rounding of a sum of squares."""
    for Lk in (1, 100, 4096, 70000):
        k = make_qkv(2, 3, Lk, d, torch.bfloat16, seed=Lk + d, device="cuda")[1]
        k[0, 1] *= 4.0                # heads with different maxima (powers of two: exact)
        k[1, 2, Lk // 2] *= 16.0
        got = binding.key_norm_max(k).double().cpu()
        ref = k.double().norm(dim=-1).amax(dim=-1).cpu()
        assert torch.allclose(got, ref, rtol=1e-5, atol=0.0), (Lk, (got / ref - 1).abs().max())


def test_key_norm_max_edge_cases(cuda):
    """No keys give 0; a key holding inf or NaN gives +inf for its head and no other."""
    assert torch.equal(binding.key_norm_max(torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device="cuda")),
                       torch.zeros(1, 2, device="cuda"))
    k = make_qkv(1, 3, 512, 128, torch.bfloat16, seed=5, device="cuda")[1]
    k[0, 1, 7, 3] = float("inf")
    k[0, 2, 300, 0] = float("nan")
    got = binding.key_norm_max(k).cpu()
    assert torch.isfinite(got[0, 0]) and got[0, 1] == float("inf") and got[0, 2] == float("inf")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_partial_fold_with_key_bound_matches_oracle(cuda, causal, d):
    """Two KV chunks folded into one state with their ra_key_norm_max bounds, on the tight ramp
    (keys nearly parallel to the queries, scores rising 17.5 log2 units): the folding kernel
    keeps the first tile's max where the bound allows. Also with no bound, and with one larger
    than the true norms (still a valid bound)."""
    from sequence_softmax_b200.inputs import ramp_qkv
    N = 2048
    q, k, v = ramp_qkv(N, d, 2.5, seed=9, device="cuda", spread=0.05)
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), d ** -0.5, causal)
    for mode in ("bound", "none", "loose"):
        st_o = torch.zeros(1, 1, N, d, device="cuda")
        st_l = torch.full((1, 1, N), float("-inf"), device="cuda")
        for c0 in (0, N // 2):
            kc, vc = k[:, :, c0:c0 + N // 2].contiguous(), v[:, :, c0:c0 + N // 2].contiguous()
            kmax = None
            if mode != "none":
                kmax = binding.key_norm_max(kc)
                if mode == "loose":
                    kmax = kmax * 3.0
            binding.partial_fold(q, kc, vc, st_o, st_l, causal=causal, k_tok0=c0, k_norm_max=kmax)
        assert binding.get_device_error() == binding.RA_OK
        compare(to_np(st_o), to_np(st_l), o_ref, lse_ref, "bf16", f"{mode} causal={causal} d={d}")
