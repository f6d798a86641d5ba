"""ra_merge on the GPU against the oracle's lse merge (fp64), through the C-ABI."""

import numpy as np
import pytest
import torch

import oracle
from sequence_softmax_b200 import binding

from .parity import to_np

pytestmark = pytest.mark.gpu


def _parts(n, rows, d, seed, neg_inf_frac=0.01, all_empty_rows=()):
    g = torch.Generator(device="cuda").manual_seed(seed)
    o = torch.randn(n, rows, d, device="cuda", generator=g)
    lse = torch.randn(n, rows, device="cuda", generator=g) + 7.0
    mask = torch.rand(n, rows, device="cuda", generator=g) < neg_inf_frac
    lse = lse.masked_fill(mask, float("-inf"))
    for r in all_empty_rows:
        lse[:, r] = float("-inf")
    return o, lse


@pytest.mark.parametrize("n,rows,d", [(1, 33, 128), (2, 1000, 128), (3, 257, 64), (16, 129, 128),
                                      (33, 40, 132), (64, 17, 4), (2, 1, 8)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_merge_matches_oracle(cuda, n, rows, d, out_dtype):
    o, lse = _parts(n, rows, d, seed=n * 1000 + rows, all_empty_rows=(0,) if rows > 1 else ())
    out, L = binding.merge(o, lse, out_dtype=out_dtype)
    assert binding.get_device_error() == binding.RA_OK
    o_ref, L_ref = oracle.merge(to_np(o), to_np(lse))
    got = to_np(out)
    tol = 1e-5 if out_dtype == torch.float32 else 2e-2
    assert np.max(np.abs(got - o_ref)) <= tol
    if out_dtype == torch.bfloat16:
        assert np.mean(np.abs(got - o_ref)) <= 2e-3
    Lg = to_np(L)
    fin = np.isfinite(L_ref)
    assert np.array_equal(np.isfinite(Lg), fin)
    assert np.max(np.abs(Lg[fin] - L_ref[fin])) <= 1e-5
    if rows > 1:
        assert np.all(got[0] == 0.0) and np.isneginf(Lg[0])


def test_merge_n1_is_identity(cuda):
    o, lse = _parts(1, 500, 128, seed=5, neg_inf_frac=0.0)
    out, L = binding.merge(o, lse, out_dtype=torch.float32)
    torch.testing.assert_close(out, o[0], rtol=0, atol=1e-6)
    torch.testing.assert_close(L, lse[0], rtol=0, atol=1e-6)


def test_merge_part_order_invariance(cuda):
    o, lse = _parts(8, 300, 128, seed=9)
    perm = torch.randperm(8, generator=torch.Generator().manual_seed(1)).cuda()
    a, La = binding.merge(o, lse, out_dtype=torch.float32)
    b, Lb = binding.merge(o[perm].contiguous(), lse[perm].contiguous(), out_dtype=torch.float32)
    torch.testing.assert_close(a, b, rtol=0, atol=1e-5)
    torch.testing.assert_close(La, Lb, rtol=0, atol=1e-5, equal_nan=True)


def test_merge_large_rows_sampled(cuda):
    """Workload-sized merge (n = 2, rows = 8 * 2^20, d = 128, bf16 out): sampled rows vs the oracle."""
    n, rows, d = 2, 8 * (1 << 20), 128
    o, lse = _parts(n, rows, d, seed=77)
    out, L = binding.merge(o, lse, out_dtype=torch.bfloat16)
    assert binding.get_device_error() == binding.RA_OK
    idx = torch.unique(torch.cat([torch.randint(0, rows, (4096,), generator=torch.Generator().manual_seed(3)),
                                  torch.tensor([0, rows - 1])])).cuda()
    o_ref, L_ref = oracle.merge(to_np(o[:, idx]), to_np(lse[:, idx]))
    got = to_np(out[idx])
    assert np.max(np.abs(got - o_ref)) <= 2e-2 and np.mean(np.abs(got - o_ref)) <= 2e-3
    fin = np.isfinite(L_ref)
    assert np.max(np.abs(to_np(L[idx])[fin] - L_ref[fin])) <= 1e-5
