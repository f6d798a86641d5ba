"""fp64 CPU oracle for the backward pass of ring attention (test infrastructure only).

``attention_backward``
    The gradients of O = softmax(S) V, S = Q K^T * scale (causal: key j visible to query i
    iff j <= i), written out: P = exp(S - lse); dV = P^T dO; dP = dO V^T;
    D_i = sum_e dO_ie O_ie (= sum_j P_ij dP_ij); dS = P * (dP - D); dQ = dS K * scale;
    dK = dS^T Q * scale. These are the steps of the ``ring_attention_backward`` listing of
    "Ring Attention 논문 분석" (youngju.dev) with the causal mask that listing omits.
    Pinned against torch autograd of ``scaled_dot_product_attention`` in fp64, central finite
    differences on tiny inputs, and closed forms.
``ring_backward``
    The ring algorithm of that listing, step by step: position p keeps Q_p, dO_p, O_p, lse_p
    and at step s receives KV chunk (p - s) mod P; it adds dS K to its own dQ_p and returns
    the chunk's dK, dV contributions to the chunk's owner, where they are summed. (The
    listing sends them with ``dist.reduce`` to a root that differs per rank, which is not a
    valid collective; the sum at the owner is the reading taken here.) Pinned against
    ``attention_backward`` for every layout and for random visiting orders.
``partial_backward``
    One query block against one KV chunk (global tokens given by offset and stride), with
    the FINAL lse and D of the query rows as inputs: the pair's additive contributions.
    Pinned: summed over the chunks of a split it equals ``attention_backward``.
``backward_rows``
    dQ at chosen query rows and dK, dV at chosen key rows of full attention, from the same
    definition (the forward state of every query row is computed blockwise first). Pinned
    against ``attention_backward`` at those rows.
"""

from __future__ import annotations

import numpy as np

from . import ring as _fwd

NEG_INF = _fwd.NEG_INF


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _probs(q, k, scale, causal, lse, tq=None, tk=None):
    """P = exp(S - lse) for one head with the causal mask; rows with lse = -inf give 0."""
    s = _fwd._scores(q, k, scale)
    if causal:
        s = np.where(_fwd._visible(tq[:, None], tk[None, :]), s, NEG_INF)
    lse_safe = np.where(np.isfinite(lse), lse, 0.0)
    p = np.exp(s - lse_safe[:, None])
    return np.where(np.isfinite(lse)[:, None], p, 0.0)


def delta(o, do):
    """D_i = sum_e dO_ie O_ie (fp64) over the last axis."""
    return (_f64(o) * _f64(do)).sum(axis=-1)


def _grads_block(q, k, v, do, d_row, lse, scale, causal, tq, tk):
    """One query block against one KV block: (dQ contribution, dK contribution, dV contribution)."""
    p = _probs(q, k, scale, causal, lse, tq, tk)
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - d_row[:, None])
    return (ds @ k) * scale, (ds.T @ q) * scale, dv


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Gradients (dQ, dK, dV) of exact softmax attention, fp64, tokens in natural order.

    q [B,H,N,d], k [B,H,Nk,d], v [B,H,Nk,dv], do [B,H,N,dv]. O and lse are recomputed with
    the forward oracle's definition.
    """
    B, H, N, _ = q.shape
    Nk = k.shape[2]
    o, lse = _fwd.attention(q, k, v, scale, causal)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    tq = np.arange(N)
    tk = np.arange(Nk)
    for b in range(B):
        for h in range(H):
            gq, gk, gv = _grads_block(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h]),
                                      delta(o[b, h], do[b, h]), lse[b, h], scale, causal, tq, tk)
            dq[b, h], dk[b, h], dv[b, h] = gq, gk, gv
    return dq, dk, dv


def ring_backward(q, k, v, do, scale: float, causal: bool, n_chunks: int, layout: str, order=None):
    """The ring backward: per position, dQ accumulated locally, dK/dV summed at the owner."""
    B, H, N, _ = q.shape
    P = n_chunks
    pos = _fwd.layout_positions(layout, N, P)
    o, lse = _fwd.ring_forward(q, k, v, scale, causal, n_chunks, layout)
    dd = delta(o, do)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            qh, kh, vh, doh = _f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h])
            for p in range(P):
                tq = pos[p]
                for s in range(P):
                    c = (p - s) % P if order is None else int(order[p][s])
                    tk = pos[c]
                    if causal and _fwd.chunk_class(tq, tk) == "skip":
                        continue
                    gq, gk, gv = _grads_block(qh[tq], kh[tk], vh[tk], doh[tq], dd[b, h, tq], lse[b, h, tq],
                                              scale, causal, tq, tk)
                    dq[b, h, tq] += gq
                    dk[b, h, tk] += gk   # returned to the owner of chunk c and summed there
                    dv[b, h, tk] += gv
    return dq, dk, dv


def partial_backward(q, k, v, do, lse, d_row, scale: float, causal: bool, q_tok0: int = 0, q_tok_stride: int = 1,
                     k_tok0: int = 0, k_tok_stride: int = 1):
    """(dQ, dK, dV) contributions of one query block [B,H,Lq,d] against one KV chunk [B,H,Lk,d].

    lse and d_row [B,H,Lq] are the query rows' final log-sum-exp and D. Query row i has token
    q_tok0 + q_tok_stride * i, key row j has k_tok0 + k_tok_stride * j.
    """
    B, H, Lq, _ = q.shape
    Lk = k.shape[2]
    tq = q_tok0 + q_tok_stride * np.arange(Lq)
    tk = k_tok0 + k_tok_stride * np.arange(Lk)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = _grads_block(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h]),
                                                        _f64(d_row[b, h]), _f64(lse[b, h]), scale, causal, tq, tk)
    return dq, dk, dv


def backward_rows(q, k, v, do, scale: float, causal: bool, q_rows, k_rows, heads=None):
    """dQ at query rows q_rows and (dK, dV) at key rows k_rows, tokens in natural order.

    heads: list of (b, h) pairs to evaluate (default: all). Returns dq [len(heads), |q_rows|, d],
    dk, dv [len(heads), |k_rows|, d] in fp64.
    """
    B, H, N, d = q.shape
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    q_rows = np.asarray(q_rows)
    k_rows = np.asarray(k_rows)
    tq_all = np.arange(N)
    dq = np.zeros((len(heads), len(q_rows), d))
    dk = np.zeros((len(heads), len(k_rows), d))
    dv = np.zeros((len(heads), len(k_rows), v.shape[-1]))
    for n, (b, h) in enumerate(heads):
        qh, kh, vh, doh = _f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h])
        if len(k_rows) == 0:
            # dQ rows need the forward state of those rows only
            o, lse = _fwd.attention(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], scale, causal,
                                    rows=q_rows)
            o, lse = o[0, 0], lse[0, 0]
            dq[n] = _grads_block(qh[q_rows], kh, vh, doh[q_rows], delta(o, doh[q_rows]), lse, scale, causal, q_rows,
                                 tq_all)[0]
            continue
        o, lse = _fwd.attention(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], scale, causal)
        o, lse = o[0, 0], lse[0, 0]
        dd = delta(o, doh)
        # dQ rows: query rows against every key
        dq[n] = _grads_block(qh[q_rows], kh, vh, doh[q_rows], dd[q_rows], lse[q_rows], scale, causal, q_rows,
                             tq_all)[0]
        # dK, dV rows: every query against the chosen keys
        _, dk[n], dv[n] = _grads_block(qh, kh[k_rows], vh[k_rows], doh, dd, lse, scale, causal, tq_all, k_rows)
    return dq, dk, dv
