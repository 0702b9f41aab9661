"""The CPU oracle against facts the pages and mathematics fix (no GPU)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    pin(oracle.load())


def test_empty_and_degenerate_sizes():
    import numpy as np
    # L = 0: y is empty and h_last is h0
    h0 = np.arange(6.0).reshape(1, 2, 3)
    z = np.zeros((1, 2, 0))
    y, h = oracle.scan_fwd(z, z, -np.ones((2, 3)), np.zeros((1, 3, 0)), np.zeros((1, 3, 0)),
                           None, None, None, True, h0)
    assert y.shape == (1, 2, 0)
    assert np.array_equal(h, h0)
    # batch = 0
    y, h = oracle.scan_fwd(np.zeros((0, 2, 4)), np.zeros((0, 2, 4)), -np.ones((2, 3)),
                           np.zeros((0, 3, 4)), np.zeros((0, 3, 4)))
    assert y.shape == (0, 2, 4) and h.shape == (0, 2, 3)
