"""The input generators do what their recipes say (CPU, no attention arithmetic)."""

import numpy as np
import torch

from sequence_softmax_b200.inputs import RAMP_BLOCK, make_qkv, ramp_qkv


def test_make_qkv_is_seeded():
    a = make_qkv(1, 2, 64, 16, torch.bfloat16, seed=3)
    b = make_qkv(1, 2, 64, 16, torch.bfloat16, seed=3)
    c = make_qkv(1, 2, 64, 16, torch.bfloat16, seed=4)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], c[0])


def _block_maxima_log2(q, k):
    """Per query row, the largest score of every key block, in log2 units at scale d^-1/2."""
    qq = q[0, 0].double().numpy()
    kk = k[0, 0].double().numpy()
    d = qq.shape[1]
    s = qq @ kk.T * d ** -0.5 / np.log(2.0)
    nb = kk.shape[0] // RAMP_BLOCK
    return s[:, : nb * RAMP_BLOCK].reshape(qq.shape[0], nb, RAMP_BLOCK).max(axis=2)


def test_ramp_moves_the_running_max_at_every_block():
    """With jump 10 every block's largest score exceeds the previous block's by more than 8
    log2 units for every row; with jump 6 the running max moves by less than 8 at each
    block but by more than 8 over two blocks."""
    for jump, lo, hi in ((10.0, 8.0, None), (6.0, 3.0, 8.0)):
        q, k, _ = ramp_qkv(1024, 128, jump, seed=1)
        step = np.diff(_block_maxima_log2(q, k), axis=1)
        assert step.min() > lo, (jump, step.min())
        if hi is not None:
            assert step.max() < hi, (jump, step.max())
            assert (step[:, 1:] + step[:, :-1]).min() > 8.0


def test_tight_ramp_reaches_the_max_skip_regime():
    """The small-spread ramp of the max-skip GPU tests: for every row the Cauchy-Schwarz bound
    |q| max|k| d^-1/2 log2(e), rounded up as the forward rounds it, lies within 22 log2 units
    of the first key block's row max (so the forward keeps that max from the second tile on,
    under its 24-unit limit), and the last block's row max is more than 8 above the first
    (so exponentials pass 2^8, where the conditional rescale alone would have moved m)."""
    for d in (64, 128):
        q, k, _ = ramp_qkv(1024, d, 2.5, seed=3, spread=0.05)
        qq, kk = q[0, 0].double().numpy(), k[0, 0].double().numpy()
        sl2 = d ** -0.5 / np.log(2.0)
        bound = np.linalg.norm(qq, axis=1) * np.linalg.norm(kk, axis=1).max() * sl2 * (1 + 2.0 ** -8) + 2.0 ** -8
        bm = _block_maxima_log2(q, k)
        assert (bound - bm[:, 0]).max() < 22.0
        assert (bm[:, -1] - bm[:, 0]).min() > 8.0
