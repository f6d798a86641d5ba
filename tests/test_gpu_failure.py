"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies runs
out, the kernel records RA_ERR_TIMEOUT in the device error word and returns, the host reads
the status, and the context keeps working (a normal ring forward afterwards still matches
the oracle)."""

import pytest
import torch

import oracle
from sequence_softmax_b200 import binding
from sequence_softmax_b200.inputs import make_qkv

from .parity import compare, to_np

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared(cuda):
    assert binding.get_device_error() == binding.RA_OK
    assert binding.selftest_wait_timeout(50_000_000) == binding.RA_ERR_TIMEOUT
    assert binding.get_device_error() == binding.RA_OK  # reading clears the word


def test_error_recorded_on_one_stream_is_read_on_another(cuda):
    """The error word belongs to the device: a timeout that a kernel on stream A records is
    reported by a read on stream B once A has finished, and only once."""
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    assert binding.get_device_error() == binding.RA_OK
    assert binding.selftest_wait_timeout(20_000_000, stream=a, read=False) == binding.RA_OK
    a.synchronize()
    assert binding.get_device_error(b) == binding.RA_ERR_TIMEOUT
    assert binding.get_device_error(b) == binding.RA_OK


def test_context_usable_after_timeout(cuda):
    assert binding.selftest_wait_timeout(20_000_000) == binding.RA_ERR_TIMEOUT
    q, k, v = make_qkv(1, 2, 1024, 128, torch.bfloat16, seed=3, device="cuda")
    o, lse = binding.ring_forward(q, k, v, 4, True, "zigzag")
    assert binding.get_device_error() == binding.RA_OK
    o_ref, lse_ref = oracle.attention(to_np(q), to_np(k), to_np(v), 128 ** -0.5, True)
    compare(to_np(o), to_np(lse), o_ref, lse_ref, "bf16", "after timeout")


def test_selftest_rejects_bad_limits(cuda):
    with pytest.raises(binding.RaError):
        binding.selftest_wait_timeout(10)
