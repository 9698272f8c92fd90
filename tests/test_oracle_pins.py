"""The fp64 oracle against closed forms, brute force and structure (no GPU)."""
import pytest

import oracle
from bwd_pins import BWD_PINS
from conv1d_pins import CONV_PINS
from oracle_pins import ALL_PINS


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)


@pytest.mark.parametrize("pin", CONV_PINS, ids=lambda f: f.__name__)
def test_conv_pin(pin, lib):
    pin(lib)


@pytest.mark.parametrize("pin", BWD_PINS, ids=lambda f: f.__name__)
def test_bwd_pin(pin, lib):
    pin(lib)
