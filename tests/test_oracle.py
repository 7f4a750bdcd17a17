"""The oracle against its pins (CPU only).  Each pin is described in oracle_pins.py."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    pin(lib)


def test_rejects_bad_shapes(lib):
    import numpy as np
    x = np.zeros((1, 4, 5, 5))
    with pytest.raises(ValueError):
        oracle.conv2d(x, np.zeros((2, 3, 3, 3)), None, lib=lib)        # C_in mismatch
    with pytest.raises(ValueError):
        oracle.conv2d(x, np.zeros((3, 2, 3, 3)), None, groups=2, lib=lib)  # C_out % groups
    with pytest.raises(ValueError):
        oracle.conv2d(x, np.zeros((2, 4, 7, 7)), None, lib=lib)        # kernel larger than input
    with pytest.raises(ValueError):
        oracle.out_size(5, 3, stride=0)


def test_threads(lib):
    assert oracle.num_threads(lib) >= 1
