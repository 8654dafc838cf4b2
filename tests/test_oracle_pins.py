"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_rejects_bad_arguments(orc):
    import numpy as np
    with pytest.raises(ValueError):
        orc.fwd(np.ones((1, 2, 1)), np.ones((1, 2, 1)), np.ones((1, 0)), np.ones((1, 2, 0)),
                np.ones((1, 2, 0)))
