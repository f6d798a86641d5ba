"""Plant plausible mistakes in the oracle (on the CPU) and check that some pin catches each.

This shows that the pins constrain every part of the oracle: a dropped term, a wrong
sign or index, a transposed operand or an off-by-one mask must make a pin fail.
"""

import numpy as np
import pytest

from oracle import ring as A

from .oracle_pins import ALL_PINS

NEG_INF = A.NEG_INF


def _scale_squared(q, k, scale):
    return (q @ k.T) * scale * scale


def _keys_transposed_with_queries(q, k, scale):
    # uses the query block where the key block belongs (shapes agree for square blocks)
    return (k @ q.T).T * scale if q.shape == k.shape else (q @ k.T) * scale * 1.0001


def _strict_mask(tq, tk):
    return tk < tq


def _mask_wrong_direction(tq, tk):
    return tk >= tq


def _no_normalisation(s, v):
    o, lse = _REAL["_softmax_rows"](s, v)
    m = s.max(axis=1)
    m = np.where(np.isfinite(m), m, 0.0)
    l = np.exp(s - m[:, None]).sum(axis=1)
    return o * l[:, None], lse


def _lse_drops_max(s, v):
    o, lse = _REAL["_softmax_rows"](s, v)
    m = s.max(axis=1)
    return o, np.where(np.isfinite(m), lse - m, lse)


def _update_forgets_l_correction(m, l, acc, s, v):
    m_new = np.maximum(m, s.max(axis=1))
    shift = np.where(np.isfinite(m_new), m_new, 0.0)
    corr = np.exp(m - shift)
    e = np.exp(s - shift[:, None])
    return m_new, l + e.sum(axis=1), acc * corr[:, None] + e @ v


def _update_wrong_sign(m, l, acc, s, v):
    m_new = np.maximum(m, s.max(axis=1))
    shift = np.where(np.isfinite(m_new), m_new, 0.0)
    corr = np.exp(np.where(np.isfinite(m), shift - m, -np.inf))
    e = np.exp(s - shift[:, None])
    return m_new, l * corr + e.sum(axis=1), acc * corr[:, None] + e @ v


def _zigzag_off_by_one(layout, N, P):
    pos = _REAL["layout_positions"](layout, N, P)
    if layout != "zigzag":
        return pos
    c = N // (2 * P)
    return [np.concatenate([np.arange(p * c, (p + 1) * c),
                            np.arange(((2 * P - p) % (2 * P)) * c, ((2 * P - p) % (2 * P) + 1) * c)])
            for p in range(P)]


def _striped_rotated(layout, N, P):
    pos = _REAL["layout_positions"](layout, N, P)
    if layout != "striped":
        return pos
    return [np.arange((p + 1) % P, N, P) for p in range(P)]


def _merge_unnormalised(o_parts, lse_parts):
    o = np.asarray(o_parts, dtype=np.float64)
    s = np.asarray(lse_parts, dtype=np.float64)
    m = s.max(axis=0)
    w = np.exp(s - m[None])
    return (w[..., None] * o).sum(axis=0), m + np.log(np.exp(s - m[None]).sum(axis=0))


def _chunk_class_never_skips(tq, tk):
    c = _REAL["chunk_class"](tq, tk)
    return "full" if c == "skip" else c


_REAL = {name: getattr(A, name) for name in
         ("_scores", "_visible", "_softmax_rows", "_online_update", "layout_positions", "merge",
          "chunk_class")}

MUTANTS = {
    "scale-squared": ("_scores", _scale_squared),
    "queries-for-keys": ("_scores", _keys_transposed_with_queries),
    "mask-drops-diagonal": ("_visible", _strict_mask),
    "mask-reversed": ("_visible", _mask_wrong_direction),
    "softmax-unnormalised": ("_softmax_rows", _no_normalisation),
    "lse-drops-max": ("_softmax_rows", _lse_drops_max),
    "online-l-uncorrected": ("_online_update", _update_forgets_l_correction),
    "online-correction-sign": ("_online_update", _update_wrong_sign),
    "zigzag-partner-off-by-one": ("layout_positions", _zigzag_off_by_one),
    "striped-rotated": ("layout_positions", _striped_rotated),
    "merge-unnormalised-weights": ("merge", _merge_unnormalised),
    "class-never-skips": ("chunk_class", _chunk_class_never_skips),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(A, attr, fn)
    failures = []
    for pin in ALL_PINS:
        try:
            ok, msg = pin(A)
        except Exception as e:  # a crash also counts as the pin rejecting the oracle
            ok, msg = False, f"raised {type(e).__name__}"
        if not ok:
            failures.append(pin.__name__)
    assert failures, f"no pin caught mutant {name}"
