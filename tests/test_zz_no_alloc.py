"""The backward entry point that allocates nothing (ra_ring_backward_noalloc).

It serves callers that cannot allocate device memory -- code inside another runtime whose
pool allocator owns the GPU's memory, or loops that cannot afford cudaMalloc's device-wide
synchronisation -- by using a static scratch array inside the library instead of a
workspace. These tests call it through the C-ABI twice in a row, on different problems (so
the second call starts from the first call's leftover scratch), and require each result to
equal ra_ring_backward's bit for bit: both run the same kernels on the same inputs, only the
scratch memory differs. This file is collected last on purpose.
"""

import ctypes

import pytest
import torch

from sequence_softmax_b200 import binding
from sequence_softmax_b200 import build as _build
from sequence_softmax_b200.inputs import make_qkv

CALLS = [
    # dtype, B, H, N, d, P, causal, layout, seed
    ("bf16", 1, 4, 2048, 128, 4, True, "zigzag", 31),
    ("bf16", 2, 2, 1536, 64, 3, False, "striped", 32),
    ("f32", 1, 2, 96, 32, 4, True, "contiguous", 33),
]


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return binding.load()


@pytest.mark.gpu
def test_noalloc_matches_ring_backward_on_consecutive_calls(lib, cuda):
    for kind, B, H, N, d, P, causal, layout, seed in CALLS:
        dtype = torch.float32 if kind == "f32" else torch.bfloat16
        q, k, v = make_qkv(B, H, N, d, dtype, seed=seed, device="cuda")
        do = make_qkv(B, H, N, d, dtype, seed=seed + 100, device="cuda")[0]
        o, lse = binding.ring_forward(q, k, v, P, causal, layout)
        ref = binding.ring_backward(q, k, v, o, do, lse, P, causal, layout)
        got = binding.ring_backward_noalloc(q, k, v, o, do, lse, P, causal, layout)
        assert binding.get_device_error() == binding.RA_OK
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            assert torch.equal(g, r), f"noalloc {layout} {kind}: {name} differs from ra_ring_backward"


def test_noalloc_rejects_problems_beyond_the_scratch(lib):
    """A problem whose workspace exceeds the static array is refused before any launch."""
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    need = lib.ra_ring_backward_workspace_bytes(binding.RA_BF16, 8, 32, 131072, 128)
    assert need > 64 * 1024 * 1024
    st = lib.ra_ring_backward_noalloc(fake, fake, fake, fake, fake, fake, binding.RA_BF16, 8, 32, 131072, 128, 0.088,
                                      4, 1, 0, fake, fake, fake, None)
    assert st == binding.RA_ERR_UNSUPPORTED
