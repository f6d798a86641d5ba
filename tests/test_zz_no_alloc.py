"""The backward entry point that allocates nothing (ra_ring_backward_noalloc).

It serves callers that cannot allocate device memory -- code inside another runtime whose
pool allocator owns the GPU's memory, or loops that cannot afford cudaMalloc's device-wide
synchronisation -- by using a static scratch array inside the library instead of a
workspace. These tests call it through the C-ABI twice in a row, on different problems (so
the second call starts from the first call's leftover scratch), and check each result
against ra_ring_backward's with the gradient tolerance of the other backward tests. This
file is collected last on purpose.
"""

import ctypes

import pytest
import torch

from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import make_qkv

from .parity import compare_grads, to_np

CALLS = [
    # dtype, B, H, N, d, P, causal, layout, seed
    ("bf16", 1, 4, 2048, 128, 4, True, "zigzag", 31),
    ("bf16", 2, 2, 1536, 64, 3, False, "striped", 32),
    ("f32", 1, 2, 96, 32, 4, True, "contiguous", 33),
]


@pytest.mark.gpu
def test_noalloc_matches_ring_backward_on_consecutive_calls(cuda):
    for kind, B, H, N, d, P, causal, layout, seed in CALLS:
        dtype = torch.float32 if kind == "f32" else torch.bfloat16
        q, k, v = make_qkv(B, H, N, d, dtype, seed=seed, device="cuda")
        do = make_qkv(B, H, N, d, dtype, seed=seed + 100, device="cuda")[0]
        o, lse = binding.ring_forward(q, k, v, P, causal, layout)
        ref = binding.ring_backward(q, k, v, o, do, lse, P, causal, layout)
        got = binding.ring_backward_noalloc(q, k, v, o, do, lse, P, causal, layout)
        assert binding.get_device_error() == binding.RA_OK
        compare_grads([to_np(t) for t in got], [to_np(t) for t in ref], kind, f"noalloc {layout} {kind}")


def test_noalloc_rejects_problems_beyond_the_scratch():
    """A problem whose workspace exceeds the static array is refused before any launch."""
    lib = binding.load()
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    need = lib.ra_ring_backward_workspace_bytes(binding.RA_BF16, 8, 32, 131072, 128)
    assert need > 64 * 1024 * 1024
    st = lib.ra_ring_backward_noalloc(fake, fake, fake, fake, fake, fake, binding.RA_BF16, 8, 32, 131072, 128, 0.088,
                                      4, 1, 0, fake, fake, fake, None)
    assert st == binding.RA_ERR_UNSUPPORTED
