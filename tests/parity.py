"""Helpers for GPU-vs-oracle parity tests: tolerances and comparisons.

Tolerances (stated for the fp32 and bf16 outputs of the path):
  fp32 inputs: max |O_gpu - O_ref| <= 1e-5 and max |lse_gpu - lse_ref| <= 1e-5.
  bf16 inputs: max |O_gpu - O_ref| <= 2e-2, mean <= 2e-3; max |lse_gpu - lse_ref| <= 1e-2.
The oracle computes in fp64 on exactly the tensors the GPU receives (bf16 widened).

Gradients (dQ, dK, dV) are compared relative to the reference's scale, since their size
grows with the sequence length: e_max = max|g - r| / max(max|r|, 1e-3) and
e_rms = ||g - r|| / max(||r||, 1e-3). The floor makes a gradient that vanishes analytically
(one query seeing one key: P = 1 and dS = 0) an absolute comparison.
  fp32: e_max <= 1e-5 (fp32 products and sums over at most a few thousand terms).
  bf16: e_max <= 2e-2, e_rms <= 5e-3. The kernel rounds P and dS to bf16 before the GEMMs
  that consume them (relative 2^-9 each), D is formed from the bf16-rounded forward output,
  and the gradients are rounded to bf16 once more: independent errors of about 2e-3 each,
  which average to about that in rms and reach a few times it at the worst element.
"""

from __future__ import annotations

import numpy as np
import torch

TOL = {
    "f32": dict(o_max=1e-5, o_mean=1e-5, lse_max=1e-5),
    "bf16": dict(o_max=2e-2, o_mean=2e-3, lse_max=1e-2),
}

GRAD_FLOOR = 1e-3

GRAD_TOL = {
    "f32": dict(e_max=1e-5, e_rms=1e-5),
    "bf16": dict(e_max=2e-2, e_rms=5e-3),
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


def compare_grads(got, ref, kind: str, what: str = ""):
    """Assert gradient parity for matching tuples (dQ, dK, dV); returns per-gradient stats."""
    tol = GRAD_TOL[kind]
    stats = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = np.asarray(g, dtype=np.float64)
        r = np.asarray(r, dtype=np.float64)
        assert g.shape == r.shape, f"{what} {name}: shape {g.shape} vs {r.shape}"
        assert np.all(np.isfinite(g)), f"{what} {name}: non-finite gradient"
        if r.size == 0:
            stats[name] = (0.0, 0.0)
            continue
        e_max = float(np.abs(g - r).max()) / max(float(np.abs(r).max()), GRAD_FLOOR)
        e_rms = float(np.linalg.norm(g - r)) / max(float(np.linalg.norm(r)), GRAD_FLOOR)
        stats[name] = (e_max, e_rms)
        assert e_max <= tol["e_max"], f"{what} {name}: e_max {e_max:.3e} > {tol['e_max']}"
        assert e_rms <= tol["e_rms"], f"{what} {name}: e_rms {e_rms:.3e} > {tol['e_rms']}"
    return stats
