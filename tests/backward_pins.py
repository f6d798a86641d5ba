"""Pins for the backward oracle (``oracle.backward``): each returns (ok, message).

* ``pin_autograd``: torch autograd of ``scaled_dot_product_attention`` in fp64 (library).
* ``pin_finite_differences``: central differences of sum(O * dO) on tiny inputs, computed
  with pure-Python attention (brute force), for every entry of Q, K and V.
* ``pin_closed_forms``: dO = 0 gives zero gradients; Q = 0 (uniform weights) gives
  dV_j = sum of dO over the queries that see key j, divided by each query's count.
* ``pin_ring_equals_definition``: the ring backward equals the definition for every layout,
  causal and not, and for random visiting orders.
* ``pin_partials_sum_to_definition``: partial_backward over every (query position, KV chunk)
  pair of a contiguous and a striped split, with the final lse and D, sums to the definition.
* ``pin_rows_equal_definition``: backward_rows equals the definition at the chosen rows.
"""

from __future__ import annotations

import math

import numpy as np
import torch

TOL = 1e-10


def _close(a, b, tol=TOL):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    if a.shape != b.shape:
        return False, f"shape {a.shape} vs {b.shape}"
    e = float(np.max(np.abs(a - b))) if a.size else 0.0
    return e <= tol, f"max abs err {e:.3e}"


def _all(checks):
    for ok, msg in checks:
        if not ok:
            return False, msg
    return True, "ok"


def pin_autograd(Bk):
    checks = []
    r = np.random.default_rng(11)
    for (B, H, N, d) in [(1, 1, 5, 8), (2, 2, 33, 16), (1, 2, 64, 64)]:
        q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
        for causal in (False, True):
            tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
            out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=d ** -0.5)
            out.backward(torch.tensor(do))
            gq, gk, gv = Bk.attention_backward(q, k, v, do, d ** -0.5, causal)
            checks += [_close(gq, tq.grad.numpy()), _close(gk, tk.grad.numpy()), _close(gv, tv.grad.numpy())]
    return _all(checks)


def _brute_loss(q, k, v, do, scale, causal):
    n = len(q)
    total = 0.0
    for i in range(n):
        keys = [j for j in range(len(k)) if (not causal or j <= i)]
        s = [sum(q[i][t] * k[j][t] for t in range(len(q[i]))) * scale for j in keys]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        z = sum(w)
        for e in range(len(v[0])):
            oe = sum(w[a] * v[j][e] for a, j in enumerate(keys)) / z
            total += oe * do[i][e]
    return total


def pin_finite_differences(Bk):
    checks = []
    r = np.random.default_rng(12)
    N, d, h = 5, 3, 1e-6
    for causal in (False, True):
        q, k, v, do = (r.standard_normal((1, 1, N, d)) for _ in range(4))
        gq, gk, gv = Bk.attention_backward(q, k, v, do, 0.8, causal)
        for name, x, g in (("q", q, gq), ("k", k, gk), ("v", v, gv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"q": q, "k": k, "v": v}
                args_m = {"q": q, "k": k, "v": v}
                args_p[name], args_m[name] = xp, xm
                lp = _brute_loss(args_p["q"][0, 0].tolist(), args_p["k"][0, 0].tolist(), args_p["v"][0, 0].tolist(),
                                 do[0, 0].tolist(), 0.8, causal)
                lm = _brute_loss(args_m["q"][0, 0].tolist(), args_m["k"][0, 0].tolist(), args_m["v"][0, 0].tolist(),
                                 do[0, 0].tolist(), 0.8, causal)
                num[idx] = (lp - lm) / (2 * h)
            checks.append(_close(g, num, 1e-6))
    return _all(checks)


def pin_closed_forms(Bk):
    checks = []
    r = np.random.default_rng(13)
    B, H, N, d = 1, 2, 24, 8
    q, k, v = (r.standard_normal((B, H, N, d)) for _ in range(3))
    zeros = np.zeros((B, H, N, d))
    for causal in (False, True):
        g = Bk.attention_backward(q, k, v, zeros, d ** -0.5, causal)
        checks += [_close(x, np.zeros_like(x)) for x in g]
    do = r.standard_normal((B, H, N, d))
    _, _, gv = Bk.attention_backward(zeros, k, v, do, d ** -0.5, False)
    checks.append(_close(gv, np.broadcast_to(do.mean(axis=2, keepdims=True), gv.shape)))
    _, _, gv = Bk.attention_backward(zeros, k, v, do, d ** -0.5, True)
    # query i sees keys 0..i with weight 1/(i+1): dV_j = sum_{i >= j} dO_i / (i + 1)
    w = do / np.arange(1, N + 1)[None, None, :, None]
    want = np.flip(np.cumsum(np.flip(w, axis=2), axis=2), axis=2)
    checks.append(_close(gv, want))
    return _all(checks)


def pin_ring_equals_definition(Bk):
    checks = []
    r = np.random.default_rng(14)
    B, H, N, d, P = 1, 2, 48, 8, 4
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    for causal in (False, True):
        want = Bk.attention_backward(q, k, v, do, d ** -0.5, causal)
        for layout in ("contiguous", "striped", "zigzag"):
            P_l = P // 2 if layout == "zigzag" else P
            got = Bk.ring_backward(q, k, v, do, d ** -0.5, causal, P_l, layout)
            checks += [_close(a, b) for a, b in zip(got, want)]
            order = np.stack([r.permutation(P_l) for _ in range(P_l)])
            got = Bk.ring_backward(q, k, v, do, d ** -0.5, causal, P_l, layout, order=order)
            checks += [_close(a, b) for a, b in zip(got, want)]
    return _all(checks)


def pin_partials_sum_to_definition(Bk):
    import oracle as Fw
    checks = []
    r = np.random.default_rng(15)
    B, H, N, d, P = 2, 1, 40, 8, 4
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    for causal in (False, True):
        want = Bk.attention_backward(q, k, v, do, d ** -0.5, causal)
        o, lse = Fw.attention(q, k, v, d ** -0.5, causal)
        dd = Bk.delta(o, do)
        for layout in ("contiguous", "striped"):
            got = [np.zeros_like(x) for x in want]
            for pq in range(P):
                for pk in range(P):
                    if layout == "contiguous":
                        iq, ik = np.arange(pq * N // P, (pq + 1) * N // P), np.arange(pk * N // P, (pk + 1) * N // P)
                        args = (int(iq[0]), 1, int(ik[0]), 1)
                    else:
                        iq, ik = np.arange(pq, N, P), np.arange(pk, N, P)
                        args = (pq, P, pk, P)
                    g = Bk.partial_backward(q[:, :, iq], k[:, :, ik], v[:, :, ik], do[:, :, iq], lse[:, :, iq],
                                            dd[:, :, iq], d ** -0.5, causal, *args)
                    got[0][:, :, iq] += g[0]
                    got[1][:, :, ik] += g[1]
                    got[2][:, :, ik] += g[2]
            checks += [_close(a, b) for a, b in zip(got, want)]
    return _all(checks)


def pin_rows_equal_definition(Bk):
    checks = []
    r = np.random.default_rng(16)
    B, H, N, d = 1, 3, 50, 8
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    rows_q, rows_k = np.array([0, 7, 49]), np.array([0, 1, 30, 49])
    for causal in (False, True):
        dq, dk, dv = Bk.attention_backward(q, k, v, do, d ** -0.5, causal)
        heads = [(0, 2), (0, 0)]
        gq, gk, gv = Bk.backward_rows(q, k, v, do, d ** -0.5, causal, rows_q, rows_k, heads=heads)
        for n, (b, h) in enumerate(heads):
            checks += [_close(gq[n], dq[b, h, rows_q]), _close(gk[n], dk[b, h, rows_k]), _close(gv[n], dv[b, h, rows_k])]
        gq, gk, _ = Bk.backward_rows(q, k, v, do, d ** -0.5, causal, rows_q, [], heads=heads)
        checks.append((gk.size == 0, "no key rows asked"))
        for n, (b, h) in enumerate(heads):
            checks.append(_close(gq[n], dq[b, h, rows_q]))
    return _all(checks)


ALL_BACKWARD_PINS = [pin_autograd, pin_finite_differences, pin_closed_forms, pin_ring_equals_definition,
                     pin_partials_sum_to_definition, pin_rows_equal_definition]
