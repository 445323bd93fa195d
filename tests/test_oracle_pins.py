"""The fp64 oracle against its pins (no GPU): hand-worked examples, closed
forms, exact-integer library routines, brute force and the method's identities."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(oracle_mod, pin):
    pin(oracle_mod, None)


def test_rejects_bad_arguments(oracle_mod):
    import numpy as np
    q = np.zeros((4, 1, 2), np.uint16)
    with pytest.raises(ValueError):
        oracle_mod.recurrent(q, q, q, np.array([0, 3], np.int32))      # does not end at T
    with pytest.raises(ValueError):
        oracle_mod.recurrent(q, q, q, np.array([0, 3, 2, 4], np.int32))  # decreasing
    with pytest.raises(ValueError):
        oracle_mod.recurrent(q, q, q, np.array([1, 4], np.int32))      # does not start at 0
    with pytest.raises(ValueError):
        oracle_mod.blocked(q, q, q, np.array([0, 4], np.int32), 0)     # block 0
    with pytest.raises(ValueError):
        oracle_mod.recurrent(q, q, q, np.array([0, 4], np.int32), heads=[1])  # head out of range
