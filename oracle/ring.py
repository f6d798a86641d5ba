"""fp64 CPU oracle: exact softmax attention, its partial states, their merge, and the ring.

Test infrastructure only (see the package docstring for who may import it). Plain
NumPy in float64, no blocking or fusion beyond what each definition states; the
only library primitives used are matrix products, ``exp``, ``log`` and ``max``.

What each function computes, and what pins it (the pins live in
``tests/test_oracle.py`` and ``tests/test_oracle_mutations.py``):

``attention``
    The definition: S = Q K^T * scale; causal keeps key token j for query token i
    iff j <= i (the ``ring_attention_causal_step`` listing masks ``triu(diagonal=1)``,
    i.e. keeps the diagonal); O = softmax_row(S) V; lse = m + log sum exp(S - m)
    (gpumode lecture 013 notes, log-sum-exp passage). Pinned against torch's
    ``scaled_dot_product_attention`` in fp64, closed forms (Q = 0, constant V,
    causal row 0) and pure-Python brute force.
``partial``
    One query block against one KV chunk with explicit global token positions,
    returned in normalised form (O_partial = acc / l, lse = m + log l); a row with
    no visible key gives O = 0 and lse = -inf. The listing
    ``ring_attention_causal_step`` returns the unnormalised triple
    (sum exp(S - m) V, m, sum exp(S - m)); the two forms carry the same information.
    Pinned by: partials over every chunk, merged, reproduce ``attention``.
``merge``
    The lse associativity lse(x) = lse([lse(x1), lse(x2)]) (lecture 013 notes),
    applied to partial outputs: L = lse over parts, O = sum_i exp(lse_i - L) O_i.
    Pinned against ``scipy.special.logsumexp`` and against ``attention``.
``layout_positions``
    Token-to-position maps: contiguous (token chunks in order, as the long-context
    data collator of the youngju.dev post splits them), striped (token t on
    position t mod P; lecture 013 notes, first remedy for causal imbalance) and
    zig-zag (position p holds chunks p and 2P-1-p of 2P; "Context Parallelism"
    card, causal imbalance section, with the chunk assignment this build takes).
    Pinned by exact-partition checks and by layout invariance of ``ring_forward``.
``ring_forward``
    The ring algorithm step by step: position p keeps its query block; at step s
    it folds KV chunk (p - s) mod P into the running state (m, l, o) with the
    online-softmax update of the ``blockwise_attention`` / ``ring_attention_forward``
    listings, skipping chunks that are wholly in the future and masking the rest
    elementwise. Pinned against ``attention`` for every layout and for random
    visiting orders (the result must not depend on the order).
``toy_ring_unstabilised``
    The 4-device simulation of the glossary's "How Ring Attention works" section:
    numerator and denominator sums of exp(q k^T / sqrt(dim)) with no max
    subtraction. The page prints that it matches full attention within 1e-5 on
    torch seed 0 inputs of shape (3, 32, 16); ``tests/golden/toy_ring.json`` holds
    that printed outcome.
"""

from __future__ import annotations

import numpy as np

NEG_INF = float("-inf")

LAYOUTS = ("contiguous", "striped", "zigzag")


# --------------------------------------------------------------------------------------
# Small building blocks (module-level so that mutation tests can plant mistakes here).
# --------------------------------------------------------------------------------------

def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _scores(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """S = Q K^T * scale for one head: q [r, d], k [c, d] -> [r, c]."""
    return (q @ k.T) * scale


def _visible(tq: np.ndarray, tk: np.ndarray) -> np.ndarray:
    """Causal visibility of key token tk to query token tq: tk <= tq (diagonal kept)."""
    return tk <= tq


def _softmax_rows(s: np.ndarray, v: np.ndarray):
    """Row softmax of masked scores s [r, c] (masked entries are -inf) applied to v [c, dv].

    Returns (O [r, dv], lse [r]). Rows with no finite score give O = 0, lse = -inf.
    """
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], NEG_INF)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe[:, None])
    l = e.sum(axis=1)
    o = e @ v
    has = l > 0
    o = np.where(has[:, None], o / np.where(has, l, 1.0)[:, None], 0.0)
    with np.errstate(divide="ignore"):
        lse = np.where(has, m_safe + np.log(np.where(has, l, 1.0)), NEG_INF)
    return o, lse


def _online_update(m, l, acc, s, v):
    """Fold one chunk's masked scores s [r, c] and values v [c, dv] into (m, l, o).

    m_new = max(m, rowmax s); corr = exp(m - m_new); l = l corr + rowsum exp(s - m_new);
    acc = acc corr + exp(s - m_new) v. A row whose maximum is still -inf uses 0 as its
    shift, so its exponentials are exactly 0 instead of NaN.
    """
    m_new = np.maximum(m, s.max(axis=1))
    shift = np.where(np.isfinite(m_new), m_new, 0.0)
    corr = np.exp(m - shift)
    e = np.exp(s - shift[:, None])
    return m_new, l * corr + e.sum(axis=1), acc * corr[:, None] + e @ v


# --------------------------------------------------------------------------------------
# The definition.
# --------------------------------------------------------------------------------------

def attention(q, k, v, scale: float, causal: bool, rows=None, row_block: int = 64):
    """Exact softmax attention in fp64, tokens in natural order.

    q [B,H,N,d], k [B,H,Nk,d], v [B,H,Nk,dv] (any float dtype; widened to fp64).
    ``rows``: optional 1-D array of query rows to evaluate (sampled mode); the result
    then has len(rows) rows in the given order. Causal requires Nk == N (self-attention).
    Returns (O [B,H,R,dv] float64, lse [B,H,R] float64, natural log).
    """
    B, H, N, _ = q.shape
    Nk = k.shape[2]
    dv = v.shape[3]
    if causal and Nk != N:
        raise ValueError("causal attention here is self-attention: Nk must equal N")
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]
    out = np.zeros((B, H, R, dv))
    lse = np.full((B, H, R), NEG_INF)
    tk_all = np.arange(Nk, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            kh = _f64(k[b, h])
            vh = _f64(v[b, h])
            for r0 in range(0, R, row_block):
                rr = rows[r0:r0 + row_block]
                qh = _f64(q[b, h][rr])
                kmax = Nk if not causal else int(min(Nk, rr.max() + 1))
                s = _scores(qh, kh[:kmax], scale)
                if causal:
                    s = np.where(_visible(rr[:, None], tk_all[None, :kmax]), s, NEG_INF)
                o, l = _softmax_rows(s, vh[:kmax])
                out[b, h, r0:r0 + len(rr)] = o
                lse[b, h, r0:r0 + len(rr)] = l
    return out, lse


def partial(q, k, v, scale: float, causal: bool,
            q_tok0: int = 0, q_tok_stride: int = 1, k_tok0: int = 0, k_tok_stride: int = 1,
            rows=None):
    """One query block against one KV chunk, normalised partial state.

    q [B,H,Lq,d], k/v [B,H,Lk,*]. Query row i has global token q_tok0 + q_tok_stride*i,
    key row j has k_tok0 + k_tok_stride*j; positions matter only when ``causal``.
    Returns (O_partial [B,H,R,dv], lse [B,H,R]); empty rows give O = 0, lse = -inf.
    """
    B, H, Lq, _ = q.shape
    Lk = k.shape[2]
    dv = v.shape[3]
    rows = np.arange(Lq, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]
    out = np.zeros((B, H, R, dv))
    lse = np.full((B, H, R), NEG_INF)
    tq = q_tok0 + q_tok_stride * rows
    tk = k_tok0 + k_tok_stride * np.arange(Lk, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            s = _scores(_f64(q[b, h][rows]), _f64(k[b, h]), scale)
            if causal:
                s = np.where(_visible(tq[:, None], tk[None, :]), s, NEG_INF)
            out[b, h], lse[b, h] = _softmax_rows(s, _f64(v[b, h]))
    return out, lse


def merge(o_parts, lse_parts):
    """lse-weighted combination of n partial states.

    o_parts [n, ..., dv], lse_parts [n, ...] -> (O [..., dv], L [...]) with
    L = log sum_i exp(lse_i) computed as max + log sum exp(lse_i - max), and
    O = sum_i exp(lse_i - L) O_i. Parts with lse = -inf get weight 0; if every part
    is -inf the row is empty: O = 0, L = -inf.
    """
    o = _f64(o_parts)
    s = _f64(lse_parts)
    m = s.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    tot = np.exp(s - m_safe[None]).sum(axis=0)
    has = tot > 0
    with np.errstate(divide="ignore"):
        L = np.where(has, m_safe + np.log(np.where(has, tot, 1.0)), NEG_INF)
    w = np.where(has[None], np.exp(s - np.where(has, L, 0.0)[None]), 0.0)
    return (w[..., None] * o).sum(axis=0), L


# --------------------------------------------------------------------------------------
# The ring, as the pages describe it (one process simulating every position).
# --------------------------------------------------------------------------------------

def layout_positions(layout: str, N: int, P: int):
    """Token indices held by each of the P virtual ring positions (a list of P int arrays).

    contiguous: position p holds tokens [p N/P, (p+1) N/P).
    striped:    position p holds tokens t with t mod P == p, in increasing order.
    zigzag:     the sequence is cut into 2P equal chunks; position p holds chunk p
                followed by chunk 2P-1-p.
    """
    if layout == "contiguous":
        if N % P:
            raise ValueError("contiguous layout needs N divisible by P")
        c = N // P
        return [np.arange(p * c, (p + 1) * c, dtype=np.int64) for p in range(P)]
    if layout == "striped":
        if N % P:
            raise ValueError("striped layout needs N divisible by P")
        return [np.arange(p, N, P, dtype=np.int64) for p in range(P)]
    if layout == "zigzag":
        if N % (2 * P):
            raise ValueError("zig-zag layout needs N divisible by 2P")
        c = N // (2 * P)
        return [np.concatenate([np.arange(p * c, (p + 1) * c, dtype=np.int64),
                                np.arange((2 * P - 1 - p) * c, (2 * P - p) * c, dtype=np.int64)])
                for p in range(P)]
    raise ValueError(f"unknown layout {layout!r}")


def chunk_class(tq: np.ndarray, tk: np.ndarray) -> str:
    """Causal class of a (query block, KV chunk) pair from their token positions.

    'skip' when every key is in the future of every query, 'full' when every key is
    visible to every query, 'diagonal' otherwise (mask elementwise).
    """
    if tk.min() > tq.max():
        return "skip"
    if tk.max() <= tq.min():
        return "full"
    return "diagonal"


def ring_forward(q, k, v, scale: float, causal: bool, n_chunks: int, layout: str,
                 order=None):
    """The ring: each position folds every KV chunk into a running (m, l, o) state.

    ``order``: optional P x P array; order[p][s] is the chunk position p visits at
    step s. Default is the ring order (p - s) mod P. Returns (O, lse) in natural
    token order, fp64.
    """
    B, H, N, _ = q.shape
    dv = v.shape[3]
    P = n_chunks
    pos = layout_positions(layout, N, P)
    out = np.zeros((B, H, N, dv))
    lse = np.full((B, H, N), NEG_INF)
    for b in range(B):
        for h in range(H):
            qh, kh, vh = _f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h])
            for p in range(P):
                tq = pos[p]
                r = tq.shape[0]
                m = np.full(r, NEG_INF)
                l = np.zeros(r)
                acc = np.zeros((r, dv))
                for s in range(P):
                    c = (p - s) % P if order is None else int(order[p][s])
                    tk = pos[c]
                    cls = chunk_class(tq, tk) if causal else "full"
                    if cls == "skip":
                        continue
                    sc = _scores(qh[tq], kh[tk], scale)
                    if cls == "diagonal":
                        sc = np.where(_visible(tq[:, None], tk[None, :]), sc, NEG_INF)
                    m, l, acc = _online_update(m, l, acc, sc, vh[tk])
                has = l > 0
                out[b, h, tq] = np.where(has[:, None], acc / np.where(has, l, 1.0)[:, None], 0.0)
                with np.errstate(divide="ignore"):
                    lse[b, h, tq] = np.where(has, m + np.log(np.where(has, l, 1.0)), NEG_INF)
    return out, lse


def toy_ring_unstabilised(q, k, v, n_devices: int):
    """The glossary's 4-device toy: q, k, v [N, dim]; no max subtraction; fp64.

    Device i keeps query block i; at step s it receives KV block (i - s) mod n and adds
    exp(q_i k_j^T / sqrt(dim)) V_j to a numerator and its row sums to a denominator.
    Returns the concatenated numerator / denominator, [N, dim].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, dim = q.shape
    blk = N // n_devices
    outs = []
    for i in range(n_devices):
        qi = q[i * blk:(i + 1) * blk]
        num = np.zeros((blk, v.shape[1]))
        den = np.zeros((blk, 1))
        for step in range(n_devices):
            j = (i - step) % n_devices
            p = np.exp(qi @ k[j * blk:(j + 1) * blk].T / np.sqrt(dim))
            num += p @ v[j * blk:(j + 1) * blk]
            den += p.sum(axis=1, keepdims=True)
        outs.append(num / den)
    return np.concatenate(outs, axis=0)
