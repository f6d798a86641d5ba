"""The FMA-pipe exp2 of the attention kernel (Cody-Waite reduction + degree-3 Remez
polynomial) against the true 2^x, on the CPU, in fp32 arithmetic step by step as the
kernel does it; and the kernel's coefficients against the generator script."""

import os
import re
import runpy

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "sequence_softmax_b200", "csrc", "attn_tc.cuh")
SCRIPT = os.path.join(ROOT, "sequence_softmax_b200", "csrc", "exp2_poly.py")


def kernel_coefficients():
    text = open(KERNEL).read()
    return [float(re.search(rf"EXP2_C{i} = ([0-9.e+-]+)f", text).group(1)) for i in range(4)]


def emulate(x, c):
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    n = (t - magic).astype(f32)
    fr = (x - n).astype(f32)
    q = (f32(c[3]) * fr + f32(c[2])).astype(f32)
    q = (q * fr + f32(c[1])).astype(f32)
    q = (q * fr + f32(c[0])).astype(f32)
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_match_generator():
    mod = runpy.run_path(SCRIPT)
    coef, err = mod["remez"]()
    assert err < 8e-5
    np.testing.assert_allclose(kernel_coefficients(), coef, rtol=1e-8)


def test_relative_error_bound():
    c = kernel_coefficients()
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 9.0, 2_000_001), rng.uniform(-125, 9, 1_000_000),
                        np.arange(-125, 10, dtype=np.float64)])
    x = x.astype(np.float32)
    got = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 8e-5, rel.max()


def test_clamp_never_wraps():
    c = kernel_coefficients()
    x = np.array([-1e30, -1000.0, -200.0, -126.6, -126.0, -125.5], dtype=np.float32)
    got = emulate(x, c)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 2.0 ** -124)
