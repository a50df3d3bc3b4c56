"""The fp64 oracle against facts that do not come from the oracle itself."""
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle)


@pytest.mark.parametrize("pin", pins.BACKWARD_PINS, ids=lambda p: p.__name__)
def test_oracle_backward_pin(pin):
    pin(oracle)


@pytest.mark.parametrize("pin", pins.DECAY_PINS + pins.FEATURE_PINS, ids=lambda p: p.__name__)
def test_oracle_decay_and_feature_pin(pin):
    pin(oracle)


@pytest.mark.parametrize("pin", pins.DECAY_BACKWARD_PINS, ids=lambda p: p.__name__)
def test_oracle_decay_backward_pin(pin):
    pin(oracle)


def test_oracle_validates_arguments():
    import numpy as np
    q = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        oracle.quadratic(q, q, q, cu_seqlens=[0, 3])      # does not end at T
    with pytest.raises(ValueError):
        oracle.recurrent(q, q, q, cu_seqlens=[0, 3, 2, 4])  # decreasing
    with pytest.raises(ValueError):
        oracle.blocked(q, q, q, 0)
    with pytest.raises(ValueError):
        oracle.decay_recurrent(q, q, q, np.array([1.5]))   # decay rate above 1
    with pytest.raises(ValueError):
        oracle.decay_state(q, q, np.array([0.5, 0.5]))     # one rate per head
