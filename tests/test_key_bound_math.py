"""The row-max skip's bound, on the CPU: by Cauchy-Schwarz every scaled score of a row is at
most |q| max|k| scale log2(e). The kernels form that product in fp32 from bf16 vectors (a
sum of squares with FMAs, a square root, two multiplies) and round it up by a relative
2^-8 and an absolute 2^-8. These tests restate that fp32 arithmetic and check that it covers
the exact scores, including keys parallel to the query, where Cauchy-Schwarz is an
equality and only the rounding margin keeps the bound above the score."""

import numpy as np
import torch

LOG2E = np.float32(1.4426950408889634)


def _bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).float().numpy()


def _norm_fp32(rows):
    """|x| of each row as the kernels compute it: fp32 sum of squares, one FMA per element."""
    out = np.empty(rows.shape[0], dtype=np.float32)
    for i, r in enumerate(rows.astype(np.float32)):
        ss = np.float32(0.0)
        for x in r:
            ss = np.float32(np.float32(x) * np.float32(x) + ss)  # fmaf(x, x, ss), one rounding
        out[i] = np.sqrt(ss, dtype=np.float32)
    return out


def _bound(q, k, scale, margin=True):
    sl2 = np.float32(np.float32(scale) * LOG2E)
    kmax = _norm_fp32(k).max()
    b = np.float32(np.float32(_norm_fp32(q) * kmax) * sl2)
    if margin:
        b = np.float32(b * np.float32(1.00390625) + np.float32(0.00390625))
    return b, sl2


def _scores(q, k, sl2):
    return (q.astype(np.float64) @ k.astype(np.float64).T) * np.float64(sl2)


def test_bound_covers_random_scores():
    rng = np.random.default_rng(0)
    for d, scale in ((64, 64 ** -0.5), (128, 128 ** -0.5), (128, 1.0), (128, 0.05)):
        q = _bf16(rng.standard_normal((64, d)) * rng.uniform(0.1, 10.0))
        k = _bf16(rng.standard_normal((256, d)) * rng.uniform(0.1, 10.0))
        b, sl2 = _bound(q, k, scale)
        s = _scores(q, k, sl2)
        assert np.all(b[:, None] >= s), (d, scale)


def test_bound_covers_parallel_keys_only_with_its_margin():
    """Keys equal to the query (up to powers of two) make the exact score equal to |q| |k|
    sl2: the fp32 product rounds either way, so the bound needs its margin; with it the bound
    clears the exact score by at least 2^-8 relative."""
    rng = np.random.default_rng(1)
    misses = 0
    for d in (64, 128):
        for trial in range(200):
            q = _bf16(rng.standard_normal((1, d)) * rng.uniform(0.5, 4.0))
            k = np.concatenate([q * 2.0 ** rng.integers(-3, 4), _bf16(rng.standard_normal((7, d)) * 0.1)])
            for scale in (d ** -0.5, 0.3):
                b, sl2 = _bound(q, k, scale)
                s = _scores(q, k, sl2)
                assert np.all(b[:, None] >= s + np.abs(s) * 2.0 ** -9)
                b0, _ = _bound(q, k, scale, margin=False)
                misses += int(np.any(b0[:, None] < s))
    assert misses > 0  # without the margin some parallel cases fall below their score


def test_skip_keeps_exponentials_below_the_limit():
    """Where a warp skips (bound <= m + 24 for every row), exp2(s sl2 - m) <= 2^24 for every
    score of every later tile, whatever the keys' directions."""
    rng = np.random.default_rng(2)
    d = 128
    skipped = 0
    for trial in range(50):
        q = _bf16(rng.standard_normal((32, d)))
        k = _bf16(rng.standard_normal((1024, d)) * rng.uniform(0.5, 2.0))
        b, sl2 = _bound(q, k, d ** -0.5)
        s = _scores(q, k, sl2)
        m = s[:, :128].max(axis=1)   # the running max after the first tile
        if np.all(b <= m + 24.0):    # the warp would keep m for the rest
            skipped += 1
            assert np.all(s[:, 128:] - m[:, None] <= 24.0)
    assert 0 < skipped < 50  # both regimes occur among these key scales
