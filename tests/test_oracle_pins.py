"""The float64 oracle against the pages' printed values, closed forms and invariants."""
import numpy as np
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle._load())


def test_rejects_nonpositive_window():
    """A window must be positive ("NNX Sliding-Window Attention", Mask before softmax:
    a positive W keeps the diagonal); W < 1 is refused rather than producing all -inf rows."""
    q = np.zeros((1, 1, 4, 2))
    for W in (0, -3):
        with pytest.raises(oracle.OracleError):
            oracle.forward(q, q, q, W)


def test_decode_rejects_negative_position():
    q = np.zeros((1, 1, 2))
    r = np.zeros((1, 1, 4, 2))
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, r, r, np.array([-1]), 4)


def test_empty_inputs():
    q = np.zeros((0, 2, 5, 3))
    assert oracle.forward(q, q, q, 2).shape == (0, 2, 5, 3)
    q = np.zeros((1, 2, 0, 3))
    assert oracle.forward(q, q, q, 2).shape == (1, 2, 0, 3)
