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


def _grads_block(q, k, v, do, o, lse, scale, causal, tq, tk):
    """One query block against one KV block: (dQ contribution, dK contribution, dV contribution)."""
    p = _probs(q, k, scale, causal, lse, tq, tk)
    dv = p.T @ do
    dp = do @ v.T
    d_row = (do * o).sum(axis=1)
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
            gq, gk, gv = _grads_block(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h]), o[b, h],
                                      lse[b, h], scale, causal, tq, tk)
            dq[b, h], dk[b, h], dv[b, h] = gq, gk, gv
    return dq, dk, dv


def ring_backward(q, k, v, do, scale: float, causal: bool, n_chunks: int, layout: str, order=None):
    """The ring backward: per position, dQ accumulated locally, dK/dV summed at the owner."""
    B, H, N, _ = q.shape
    P = n_chunks
    pos = _fwd.layout_positions(layout, N, P)
    o, lse = _fwd.ring_forward(q, k, v, scale, causal, n_chunks, layout)
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
                    gq, gk, gv = _grads_block(qh[tq], kh[tk], vh[tk], doh[tq], o[b, h, tq], lse[b, h, tq], scale,
                                              causal, tq, tk)
                    dq[b, h, tq] += gq
                    dk[b, h, tk] += gk   # returned to the owner of chunk c and summed there
                    dv[b, h, tk] += gv
    return dq, dk, dv
