"""Helpers for GPU-vs-oracle parity tests: tolerances and comparisons.

Tolerances (stated for the fp32 and bf16 outputs of the path):
  fp32 inputs: max |O_gpu - O_ref| <= 1e-5 and max |lse_gpu - lse_ref| <= 1e-5.
  bf16 inputs: max |O_gpu - O_ref| <= 2e-2, mean <= 2e-3; max |lse_gpu - lse_ref| <= 1e-2.
The oracle computes in fp64 on exactly the tensors the GPU receives (bf16 widened).
"""

from __future__ import annotations

import numpy as np
import torch

TOL = {
    "f32": dict(o_max=1e-5, o_mean=1e-5, lse_max=1e-5),
    "bf16": dict(o_max=2e-2, o_mean=2e-3, lse_max=1e-2),
}


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def compare(o_gpu, lse_gpu, o_ref, lse_ref, kind: str, what: str = ""):
    """Assert parity; returns the error statistics."""
    tol = TOL[kind]
    o = np.asarray(o_gpu, dtype=np.float64)
    err = np.abs(o - o_ref)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    stats = {"o_max": float(err.max()) if err.size else 0.0, "o_mean": float(err.mean()) if err.size else 0.0}
    assert stats["o_max"] <= tol["o_max"], f"{what}: max abs err {stats['o_max']:.3e} > {tol['o_max']}"
    assert stats["o_mean"] <= tol["o_mean"], f"{what}: mean abs err {stats['o_mean']:.3e} > {tol['o_mean']}"
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, dtype=np.float64)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin), f"{what}: lse finiteness differs"
        assert np.all(lg[~fin] == lse_ref[~fin]), f"{what}: empty rows must have lse = -inf"
        e = np.abs(lg[fin] - lse_ref[fin])
        stats["lse_max"] = float(e.max()) if e.size else 0.0
        assert stats["lse_max"] <= tol["lse_max"], f"{what}: lse err {stats['lse_max']:.3e} > {tol['lse_max']}"
    return stats
