"""The CPU oracle against its pins (closed forms, the printed formula, the
running-sum route, exact rationals, symmetries).  No GPU needed."""
import pytest

import oracle
from pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.default())


def test_invalid_arguments_rejected():
    import numpy as np
    q = np.zeros((1, 4, 1, 8), np.float32)
    c = np.ones((4, 4), np.float32)
    s = np.zeros((4, 4), np.float32)
    with pytest.raises(ValueError):
        oracle.recurrence(q, q, q, c, s, 0)
    with pytest.raises(ValueError):
        oracle.masked(q, q, q, c, s, 2, rows=np.array([4]))
    with pytest.raises(ValueError):
        oracle.recurrence(q, q, q, c[:3], s[:3], 2)
    with pytest.raises(TypeError):
        oracle.recurrence(q.astype(np.float64), q, q, c, s, 2)
