"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each pin takes the oracle module (``oracle.ring``) and returns (ok, message). The
same pins run against the real oracle (``test_oracle.py``, all must pass) and against
copies with a planted mistake (``test_oracle_mutations.py``, at least one must fail).

What each pin compares with:

* ``pin_toy_pages``: the glossary's 4-device simulation ("How Ring Attention works"):
  the page prints that the ring result matches torch's full softmax attention within
  atol 1e-5 on torch seed 0 inputs of shape (3, 32, 16); ``tests/golden/toy_ring.json``.
* ``pin_sdpa``: torch's ``scaled_dot_product_attention`` in fp64 on CPU (a library
  routine) and ``torch.logsumexp`` of the masked scores for lse.
* ``pin_closed_forms``: Q = 0 gives uniform weights (O = mean of the visible V rows,
  lse = log of their count); constant V gives that constant; causal row 0 sees only
  key 0, so O_0 = V_0 and lse_0 = q_0 . k_0 * scale.
* ``pin_bruteforce``: pure-Python loops with ``math.exp`` on tiny inputs.
* ``pin_lse_associativity``: lse(x) = lse([lse(x1), lse(x2)]) (lecture 013 notes,
  log-sum-exp passage) against ``scipy.special.logsumexp`` / ``softmax``.
* ``pin_merge_reproduces_full``: partial states of every KV chunk, merged, equal full
  attention (non-causal and causal with global token offsets).
* ``pin_order_invariance``: the ring gives the same result for any visiting order.
* ``pin_layouts``: positions partition the tokens exactly as each layout states, and
  the ring equals full attention for every layout, causal and not.
* ``pin_empty_rows``: rows with no visible key give O = 0, lse = -inf, in partial and merge.
* ``pin_sampled_rows``: sampled mode returns exactly the requested rows of the full result.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol=TOL):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.shape != b.shape:
        return False, f"shape {a.shape} vs {b.shape}"
    fin_a, fin_b = np.isfinite(a), np.isfinite(b)
    if not np.array_equal(fin_a, fin_b) or not np.array_equal(a[~fin_a], b[~fin_b]):
        return False, "non-finite entries differ"
    err = float(np.max(np.abs(a[fin_a] - b[fin_b]))) if fin_a.any() else 0.0
    return err <= tol, f"max abs err {err:.3e} (tol {tol:.1e})"


def _all(checks):
    for ok, msg in checks:
        if not ok:
            return False, msg
    return True, "ok"


def _sdpa(q, k, v, scale, causal):
    t = [torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(*t, is_causal=causal, scale=scale).numpy()


def _torch_lse(q, k, scale, causal):
    s = torch.as_tensor(np.asarray(q, np.float64)) @ torch.as_tensor(np.asarray(k, np.float64)).transpose(-1, -2)
    s = s * scale
    if causal:
        n = s.shape[-1]
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    return torch.logsumexp(s, dim=-1).numpy()


# --------------------------------------------------------------------------------------

def pin_toy_pages(A):
    """The glossary toy: ring and definition match torch full attention; the page's check passes."""
    with open(os.path.join(GOLDEN, "toy_ring.json")) as f:
        g = json.load(f)
    gen = torch.Generator().manual_seed(g["seed"])
    n, blk, dim = g["n_devices"], g["block"], g["dim"]
    q, k, v = torch.randn(3, n * blk, dim, generator=gen)
    full32 = torch.softmax(q @ k.T / dim ** 0.5, dim=-1) @ v          # the page's fp32 reference
    full64 = (torch.softmax(q.double() @ k.double().T / dim ** 0.5, dim=-1) @ v.double()).numpy()
    q4, k4, v4 = (x.view(1, 1, n * blk, dim).numpy() for x in (q, k, v))
    o_def, _ = A.attention(q4, k4, v4, dim ** -0.5, False)
    o_ring, _ = A.ring_forward(q4, k4, v4, dim ** -0.5, False, n, "contiguous")
    toy = A.toy_ring_unstabilised(q.numpy(), k.numpy(), v.numpy(), n)
    page_ok = bool(np.allclose(toy, full32.numpy(), atol=g["atol"], rtol=0))
    checks = [
        _close(o_def[0, 0], full64),
        _close(o_ring[0, 0], full64),
        _close(toy, full64, 1e-10),
        (page_ok == g["matches_full_attention"], f"page check gives {page_ok}"),
        ((blk, blk) == tuple(g["score_block_per_device"]), "block shape"),
        ((n * blk, n * blk) == tuple(g["full_score_matrix"]), "full shape"),
    ]
    return _all(checks)


def pin_sdpa(A):
    checks = []
    r = _rng(1)
    for (B, H, N, d) in [(1, 1, 1, 8), (2, 3, 7, 16), (1, 2, 33, 64), (2, 1, 64, 128)]:
        q, k, v = (r.standard_normal((B, H, N, d)) for _ in range(3))
        scale = d ** -0.5
        for causal in (False, True):
            o, lse = A.attention(q, k, v, scale, causal)
            checks.append(_close(o, _sdpa(q, k, v, scale, causal)))
            checks.append(_close(lse, _torch_lse(q, k, scale, causal)))
    # cross-attention shape (Nk != N), non-causal
    q = r.standard_normal((1, 2, 5, 16))
    k = r.standard_normal((1, 2, 11, 16))
    v = r.standard_normal((1, 2, 11, 24))
    o, lse = A.attention(q, k, v, 0.25, False)
    checks.append(_close(o, _sdpa(q, k, v, 0.25, False)))
    checks.append(_close(lse, _torch_lse(q, k, 0.25, False)))
    return _all(checks)


def pin_closed_forms(A):
    checks = []
    r = _rng(2)
    B, H, N, d = 1, 2, 40, 16
    k = r.standard_normal((B, H, N, d))
    v = r.standard_normal((B, H, N, d))
    q0 = np.zeros((B, H, N, d))
    o, lse = A.attention(q0, k, v, d ** -0.5, False)
    checks.append(_close(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape)))
    checks.append(_close(lse, np.full((B, H, N), math.log(N))))
    o, lse = A.attention(q0, k, v, d ** -0.5, True)
    prefix = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    checks.append(_close(o, prefix))
    checks.append(_close(lse, np.broadcast_to(np.log(np.arange(1, N + 1)), lse.shape)))
    q = r.standard_normal((B, H, N, d))
    c = np.full((B, H, N, d), 0.37)
    for causal in (False, True):
        o, _ = A.attention(q, k, c, d ** -0.5, causal)
        checks.append(_close(o, c))
    o, lse = A.attention(q, k, v, d ** -0.5, True)
    checks.append(_close(o[:, :, 0], v[:, :, 0]))
    checks.append(_close(lse[:, :, 0], (q[:, :, 0] * k[:, :, 0]).sum(-1) * d ** -0.5))
    return _all(checks)


def _brute(q, k, v, scale, causal):
    """Pure-Python exact attention for one head: lists of lists."""
    n, nk = len(q), len(k)
    out, lses = [], []
    for i in range(n):
        keys = [j for j in range(nk) if (not causal or j <= i)]
        s = [sum(q[i][t] * k[j][t] for t in range(len(q[i]))) * scale for j in keys]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = sum(w)
        out.append([sum(w[a] * v[j][e] for a, j in enumerate(keys)) / tot for e in range(len(v[0]))])
        lses.append(mx + math.log(tot))
    return out, lses


def pin_bruteforce(A):
    checks = []
    r = _rng(3)
    for (N, d, dv) in [(1, 4, 4), (5, 3, 6), (12, 8, 8)]:
        q, k = r.standard_normal((1, 2, N, d)), r.standard_normal((1, 2, N, d))
        v = r.standard_normal((1, 2, N, dv))
        for causal in (False, True):
            o, lse = A.attention(q, k, v, 0.7, causal)
            for h in range(2):
                bo, bl = _brute(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), 0.7, causal)
                checks.append(_close(o[0, h], np.array(bo)))
                checks.append(_close(lse[0, h], np.array(bl)))
    return _all(checks)


def pin_lse_associativity(A):
    from scipy.special import logsumexp, softmax
    checks = []
    r = _rng(4)
    for n_parts, size in [(2, 10), (2, 1000), (5, 37), (16, 4096)]:
        x = r.standard_normal(size) * 3.0
        cuts = np.sort(r.choice(np.arange(1, size), n_parts - 1, replace=False))
        parts = np.split(x, cuts)
        lse_parts = np.array([logsumexp(p) for p in parts])
        # lse(x) = lse([lse(x1), ..., lse(xn)]): merge a scalar "output" of ones per part
        _, L = A.merge(np.ones((n_parts, 1, 1)), lse_parts[:, None])
        checks.append(_close(L[0], logsumexp(x), 1e-11))
        # the notebook's intent: partial softmaxes reweighted by their share equal softmax(x)
        weights = np.exp(lse_parts - L[0])
        combined = np.concatenate([softmax(p) * w for p, w in zip(parts, weights)])
        checks.append(_close(combined, softmax(x), 1e-12))
    return _all(checks)


def pin_merge_reproduces_full(A):
    checks = []
    r = _rng(5)
    B, H, N, d = 2, 2, 48, 16
    q, k, v = (r.standard_normal((B, H, N, d)) for _ in range(3))
    scale = d ** -0.5
    for causal in (False, True):
        o_ref, lse_ref = A.attention(q, k, v, scale, causal)
        for cuts in ([16, 32], [5, 6, 40], [24]):
            bounds = [0] + cuts + [N]
            parts = [A.partial(q, k[:, :, a:b], v[:, :, a:b], scale, causal, 0, 1, a, 1)
                     for a, b in zip(bounds[:-1], bounds[1:])]
            o, lse = A.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
            checks.append(_close(o, o_ref))
            checks.append(_close(lse, lse_ref))
    # strided token positions: query rows of one striped position against another's keys
    P = 4
    for pq in range(P):
        tq = np.arange(pq, N, P)
        o_ref, lse_ref = A.attention(q, k, v, scale, True, rows=tq)
        parts = []
        for pk in range(P):
            tk = np.arange(pk, N, P)
            parts.append(A.partial(q[:, :, tq], k[:, :, tk], v[:, :, tk], scale, True, pq, P, pk, P))
        o, lse = A.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        checks.append(_close(o, o_ref))
        checks.append(_close(lse, lse_ref))
    return _all(checks)


def pin_order_invariance(A):
    checks = []
    r = _rng(6)
    B, H, N, d, P = 1, 2, 64, 8, 8
    q, k, v = (r.standard_normal((B, H, N, d)) for _ in range(3))
    for causal in (False, True):
        o_ref, lse_ref = A.attention(q, k, v, d ** -0.5, causal)
        for layout in ("contiguous", "striped", "zigzag"):
            P_l = P // 2 if layout == "zigzag" else P
            order = np.stack([r.permutation(P_l) for _ in range(P_l)])
            o, lse = A.ring_forward(q, k, v, d ** -0.5, causal, P_l, layout, order=order)
            checks.append(_close(o, o_ref))
            checks.append(_close(lse, lse_ref))
    return _all(checks)


def pin_layouts(A):
    checks = []
    N, P = 64, 4
    pos = A.layout_positions("contiguous", N, P)
    checks.append((all(np.array_equal(pos[p], np.arange(16 * p, 16 * p + 16)) for p in range(P)), "contiguous"))
    pos = A.layout_positions("striped", N, P)
    checks.append((all(set(pos[p].tolist()) == {t for t in range(N) if t % P == p} for p in range(P)), "striped"))
    pos = A.layout_positions("zigzag", N, P)
    c = N // (2 * P)
    for p in range(P):
        want = set(range(p * c, (p + 1) * c)) | set(range((2 * P - 1 - p) * c, (2 * P - p) * c))
        checks.append((set(pos[p].tolist()) == want and len(pos[p]) == 2 * c, f"zigzag position {p}"))
    for layout in ("contiguous", "striped", "zigzag"):
        allt = np.sort(np.concatenate(A.layout_positions(layout, N, P)))
        checks.append((np.array_equal(allt, np.arange(N)), f"{layout} is a partition"))
    r = _rng(7)
    q, k, v = (r.standard_normal((2, 1, N, 8)) for _ in range(3))
    for causal in (False, True):
        o_ref, lse_ref = A.attention(q, k, v, 8 ** -0.5, causal)
        for layout in ("contiguous", "striped", "zigzag"):
            o, lse = A.ring_forward(q, k, v, 8 ** -0.5, causal, P, layout)
            checks.append(_close(o, o_ref))
            checks.append(_close(lse, lse_ref))
    # chunk classes agree with brute-force visibility counts
    for layout in ("contiguous", "striped", "zigzag"):
        pos = A.layout_positions(layout, N, P)
        for a in range(P):
            for b in range(P):
                vis = (pos[b][None, :] <= pos[a][:, None])
                want = "skip" if not vis.any() else ("full" if vis.all() else "diagonal")
                checks.append((A.chunk_class(pos[a], pos[b]) == want, f"class {layout} {a},{b}"))
    return _all(checks)


def pin_empty_rows(A):
    checks = []
    r = _rng(8)
    q, k, v = (r.standard_normal((1, 1, 8, 4)) for _ in range(3))
    # keys at tokens 100..107 are all in the future of queries at tokens 0..7
    o, lse = A.partial(q, k, v, 0.5, True, 0, 1, 100, 1)
    checks.append((np.all(o == 0.0) and np.all(np.isneginf(lse)), "future-only chunk"))
    # partly visible: query token t sees keys 4..t
    o, lse = A.partial(q, k, v, 0.5, True, 0, 1, 4, 1)
    checks.append((np.all(o[0, 0, :4] == 0.0) and np.all(np.isneginf(lse[0, 0, :4])), "empty prefix rows"))
    checks.append((np.all(np.isfinite(lse[0, 0, 4:])), "non-empty rows finite"))
    o2, lse2 = A.merge(np.stack([o, np.zeros_like(o)]), np.stack([lse, np.full_like(lse, -np.inf)]))
    checks.append(_close(o2, o))
    checks.append(_close(lse2, lse))
    return _all(checks)


def pin_sampled_rows(A):
    r = _rng(9)
    q, k, v = (r.standard_normal((1, 2, 50, 8)) for _ in range(3))
    rows = np.array([49, 0, 17, 3, 33])
    checks = []
    for causal in (False, True):
        o, lse = A.attention(q, k, v, 0.3, causal)
        os_, ls_ = A.attention(q, k, v, 0.3, causal, rows=rows, row_block=2)
        checks.append(_close(os_, o[:, :, rows]))
        checks.append(_close(ls_, lse[:, :, rows]))
    return _all(checks)


ALL_PINS = [pin_toy_pages, pin_sdpa, pin_closed_forms, pin_bruteforce, pin_lse_associativity,
            pin_merge_reproduces_full, pin_order_invariance, pin_layouts, pin_empty_rows,
            pin_sampled_rows]
