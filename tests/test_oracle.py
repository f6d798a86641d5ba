"""The fp64 oracle against its pins (CPU only). Every pin must pass before any GPU result
is trusted; see ``oracle_pins.py`` for what each pin compares with."""

import numpy as np
import pytest

import oracle
from oracle import ring as A

from .oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    ok, msg = pin(A)
    assert ok, msg


def test_package_exports_same_functions():
    assert oracle.attention is A.attention
    assert oracle.ring_forward is A.ring_forward
    assert oracle.merge is A.merge


def test_layout_validation():
    with pytest.raises(ValueError):
        A.layout_positions("zigzag", 20, 4)
    with pytest.raises(ValueError):
        A.layout_positions("striped", 10, 4)
    with pytest.raises(ValueError):
        A.layout_positions("diagonal", 16, 4)


def test_causal_requires_self_attention():
    x = np.zeros((1, 1, 4, 2))
    y = np.zeros((1, 1, 5, 2))
    with pytest.raises(ValueError):
        A.attention(x, y, y, 1.0, True)
