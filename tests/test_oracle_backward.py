"""The backward oracle against its pins, and planted mistakes that some pin must catch."""

import pytest

from oracle import backward as Bk

from .backward_pins import ALL_BACKWARD_PINS


@pytest.mark.parametrize("pin", ALL_BACKWARD_PINS, ids=lambda p: p.__name__)
def test_backward_pin(pin):
    ok, msg = pin(Bk)
    assert ok, msg


_REAL = Bk._grads_block


def _no_d_term(q, k, v, do, d_row, lse, scale, causal, tq, tk):
    p = Bk._probs(q, k, scale, causal, lse, tq, tk)
    ds = p * (do @ v.T)
    return (ds @ k) * scale, (ds.T @ q) * scale, p.T @ do


def _missing_scale(q, k, v, do, d_row, lse, scale, causal, tq, tk):
    gq, gk, gv = _REAL(q, k, v, do, d_row, lse, scale, causal, tq, tk)
    return gq / scale, gk, gv


def _dv_untransposed(q, k, v, do, d_row, lse, scale, causal, tq, tk):
    gq, gk, gv = _REAL(q, k, v, do, d_row, lse, scale, causal, tq, tk)
    p = Bk._probs(q, k, scale, causal, lse, tq, tk)
    if p.shape[0] != p.shape[1]:
        return gq, gk, gv * 1.5    # only square blocks can take p @ dO; corrupt the rest plainly
    return gq, gk, p @ do


def _dk_uses_k(q, k, v, do, d_row, lse, scale, causal, tq, tk):
    gq, gk, gv = _REAL(q, k, v, do, d_row, lse, scale, causal, tq, tk)
    p = Bk._probs(q, k, scale, causal, lse, tq, tk)
    ds = p * (do @ v.T - d_row[:, None])
    return gq, (ds.T @ k) * scale, gv


def _no_causal_mask(q, k, v, do, d_row, lse, scale, causal, tq, tk):
    return _REAL(q, k, v, do, d_row, lse, scale, False, tq, tk)


MUTANTS = {"drop-D": _no_d_term, "dq-missing-scale": _missing_scale, "dv-untransposed": _dv_untransposed,
           "dk-uses-k": _dk_uses_k, "no-causal-mask": _no_causal_mask}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(Bk, "_grads_block", MUTANTS[name])
    failed = []
    for pin in ALL_BACKWARD_PINS:
        try:
            ok, _ = pin(Bk)
        except Exception:
            ok = False
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"no pin caught {name}"
